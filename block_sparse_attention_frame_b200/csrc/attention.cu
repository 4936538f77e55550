// Host side of the LVSA attention path: tensor maps, launches and the C ABI entry points
// lvsa_attention (device buffers) and lvsa_attention_host (host buffers, transfers pipelined by bands of
// heads), plus the status and test hooks declared in lvsa.h.  The kernel is in attention_kernel.cuh.
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <climits>
#include <cstdio>
#include <mutex>
#include <vector>

#include "attention_kernel.cuh"
#include "buffer_checks.h"

namespace lvsa {
// ------------------------------------------------------------------ host side
namespace {

unsigned long long g_wait_ns = 4000000000ull;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// A band of H heads out of rows of HS heads: [batch][tokens][HS*d] bf16 starting at `base`
// (the band's first head) viewed as a 3-D tensor {H*d, tokens, batch} with row pitch HS*d;
// one box = 64 columns (128 bytes, one swizzle row) x `rows` tokens (128: a whole tile; 8: a piece of a tile
// that spans two runs of frames).
bool make_map(CUtensorMap* tm, const void* base, int B, long long tokens, int H, int HS, int d, int rows = kBM) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(H) * d, static_cast<cuuint64_t>(tokens),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(HS) * d * 2, static_cast<cuuint64_t>(tokens) * HS * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

std::mutex g_attr_mu;
bool g_attr_set[2][64] = {};

template <int D>
lvsa_status launch(const KernelParams& kp, int nlaunch, int B, cudaStream_t stream, int dev) {
  using Cf = Cfg<D>;
  const int di = (D == 128) ? 1 : 0;
  {
    std::lock_guard<std::mutex> g(g_attr_mu);
    if (dev < 0 || dev >= 64) return LVSA_ERR_UNSUPPORTED;
    if (!g_attr_set[di][dev]) {
      if (cudaFuncSetAttribute(lvsa_attention_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::kSmemBytes) != cudaSuccess)
        return LVSA_ERR_CUDA;
      g_attr_set[di][dev] = true;
    }
  }
  dim3 grid(static_cast<unsigned>(nlaunch), static_cast<unsigned>(kp.H), static_cast<unsigned>(B));
  lvsa_attention_kernel<D><<<grid, kThreads, Cf::kSmemBytes, stream>>>(kp);
  return cudaGetLastError() == cudaSuccess ? LVSA_OK : LVSA_ERR_CUDA;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace
}  // namespace lvsa

namespace lvsa {
namespace {

// Checks shared by the attention entry points (no CUDA call).
lvsa_status check_sizes(int L, int T, int P, int heads, int d, int batch, float scale, int text_tokens = 0) {
  if (T < 1 || P < 1 || heads < 1 || batch < 1 || L < 1 || L > T || text_tokens < 0) return LVSA_ERR_INVALID_ARG;
  if (heads > 65535 || batch > 65535) return LVSA_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * P + text_tokens > INT_MAX) return LVSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return LVSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LVSA_ERR_UNSUPPORTED;
  if (T > kMaxT) return LVSA_ERR_UNSUPPORTED;
  return LVSA_OK;
}

lvsa_status check_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return LVSA_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess) return LVSA_ERR_CUDA;
  return major == 10 ? LVSA_OK : LVSA_ERR_UNSUPPORTED;
}

// Where a launch writes its output: token ranges of the frame-major sequence, one buffer each, every
// buffer [batch][tokens of its range][head_stride][d], this launch's heads starting at head0.
struct Route {
  int nchunks = 1;
  int start[kMaxChunks + 1] = {};
  void* out[kMaxChunks] = {};
  int head_stride = 1;
  int head0 = 0;
  int routed = 0;
};

Route one_buffer(void* out, long long tokens, int head_stride) {
  Route r;
  r.start[1] = static_cast<int>(tokens);
  r.out[0] = out;
  r.head_stride = head_stride;
  return r;
}

// Query blocks of a launch over T*P video tokens and ntext text tokens (256-row blocks over the whole
// sequence when frames hold at least 256 tokens, else blocks inside each frame; text rows after them).
struct Blocks {
  int straddle, qblocks;
  long long nvblocks, nblocks;
};
Blocks query_blocks(int T, int P, int ntext) {
  constexpr int kRows = kQTiles * kBM;
  Blocks bl;
  bl.qblocks = (P + kRows - 1) / kRows;
  bl.straddle = P >= kRows ? 1 : 0;
  bl.nvblocks = bl.straddle ? (static_cast<long long>(T) * P + kRows - 1) / kRows : static_cast<long long>(T) * bl.qblocks;
  bl.nblocks = bl.nvblocks + (ntext + kRows - 1) / kRows;
  return bl;
}

// One launch over `heads` heads whose input rows hold `in_stride` heads; q, k, v point at the band's
// first head.  A joint sequence holds `ntext` text tokens after the T*P video tokens.  The launch covers
// query blocks [block0, block0 + nlaunch) (nlaunch < 0: every block).  Arguments are already validated.
lvsa_status launch_band(const void* q, const void* k, const void* v, const int32_t* lists, int L, int T, int P,
                        int heads, int in_stride, int d, int batch, float scale, const Route& route,
                        cudaStream_t st, int dev, int ntext = 0, int block0 = 0, int nlaunch = -1) {
  // frames of at least 256 tokens: query blocks of 256 rows run over the whole
  // sequence (a block may hold the end of one frame and the start of the next);
  // shorter frames: blocks stay inside a frame.  Text rows take blocks of their own.
  const Blocks bl = query_blocks(T, P, ntext);
  const int qblocks = bl.qblocks, straddle = bl.straddle;
  const long long nvblocks = bl.nvblocks, nblocks = bl.nblocks;
  if (nblocks > INT_MAX) return LVSA_ERR_INVALID_ARG;
  if (nlaunch < 0) {
    block0 = 0;
    nlaunch = static_cast<int>(nblocks);
  }
  if (block0 < 0 || nlaunch < 1 || block0 + static_cast<long long>(nlaunch) > nblocks) return LVSA_ERR_INVALID_ARG;
  KernelParams kp;
  const long long tokens = static_cast<long long>(T) * P + ntext;
  if (!make_map(&kp.tm_q, q, batch, tokens, heads, in_stride, d) ||
      !make_map(&kp.tm_k, k, batch, tokens, heads, in_stride, d) ||
      !make_map(&kp.tm_v, v, batch, tokens, heads, in_stride, d) ||
      !make_map(&kp.tm_k8, k, batch, tokens, heads, in_stride, d, 8) ||
      !make_map(&kp.tm_v8, v, batch, tokens, heads, in_stride, d, 8))
    return LVSA_ERR_CUDA;
  kp.pack = (P % 8 == 0 && ntext == 0) ? 1 : 0;
  kp.lists = lists;
  kp.T = T;
  kp.P = P;
  kp.ntext = ntext;
  kp.nvblocks = static_cast<int>(nvblocks);
  kp.H = heads;
  kp.HS = route.head_stride;
  kp.head0 = route.head0;
  kp.nchunks = route.nchunks;
  kp.routed = route.routed;
  for (int c = 0; c <= kMaxChunks; ++c) kp.chunk_start[c] = route.start[c <= route.nchunks ? c : route.nchunks];
  for (int c = 0; c < kMaxChunks; ++c)
    kp.out_chunk[c] = static_cast<__nv_bfloat16*>(c < route.nchunks ? route.out[c] : nullptr);
  kp.L = L;
  kp.qblocks = qblocks;
  kp.straddle = straddle;
  kp.nblocks = static_cast<int>(nblocks);
  kp.block0 = block0;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  kp.scale_log2 = sc * 1.4426950408889634f;
  kp.wait_cycles = wait_budget_cycles(g_wait_ns);
  return d == 128 ? launch<128>(kp, nlaunch, batch, st, dev) : launch<64>(kp, nlaunch, batch, st, dev);
}

// Streams and events of the host-buffer path, created once per device and kept: one upload and one
// readback stream, and two streams the band kernels alternate on, so that a band's CTAs start on the
// SMs the previous band's last wave leaves free.
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr, k[2] = {nullptr, nullptr};
  std::vector<cudaEvent_t> ev;  // 2 per launch (a band, or a piece of one) + 2
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];

lvsa_status pipe_for(int dev, int bands, HostPipe** out) {
  if (dev < 0 || dev >= 64) return LVSA_ERR_UNSUPPORTED;
  HostPipe& hp = g_pipe[dev];
  if (!hp.h2d && cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess) return LVSA_ERR_CUDA;
  if (!hp.d2h && cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess) return LVSA_ERR_CUDA;
  for (int i = 0; i < 2; ++i)
    if (!hp.k[i] && cudaStreamCreateWithFlags(&hp.k[i], cudaStreamNonBlocking) != cudaSuccess) return LVSA_ERR_CUDA;
  const size_t need = 2 * static_cast<size_t>(bands) + 2;  // `bands`: launches the call may make
  while (hp.ev.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return LVSA_ERR_CUDA;
    hp.ev.push_back(e);
  }
  *out = &hp;
  return LVSA_OK;
}

bool disjoint(const void* a, const void* b, size_t bytes) { return ranges_disjoint(a, bytes, b, bytes); }

// A named range on a profiler's host timeline (NVTX).  With no profiler attached a push or pop is a call
// that returns at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  NvtxRange(const char* what, int band) {
    char buf[48];
    std::snprintf(buf, sizeof(buf), "%s %d", what, band);
    nvtxRangePushA(buf);
  }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

PeerOps runtime_peer_ops() { return PeerOps{cudaDeviceCanAccessPeer, cudaDeviceEnablePeerAccess, cudaGetLastError}; }

}  // namespace
}  // namespace lvsa

// ------------------------------------------------------------------ C ABI
extern "C" lvsa_status lvsa_attention(const void* q, const void* k, const void* v, const int32_t* lists, int L,
                                      int T, int tokens_per_frame, int heads, int d, int batch, float scale,
                                      void* out, void* stream) {
  using namespace lvsa;
  const int P = tokens_per_frame;
  if (!q || !k || !v || !lists || !out) return LVSA_ERR_INVALID_ARG;
  if (T < 1 || P < 1 || heads < 1 || batch < 1 || L < 1 || L > T) return LVSA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return LVSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lists) & 3u))
    return LVSA_ERR_INVALID_ARG;
  const lvsa_status cs = check_sizes(L, T, P, heads, d, batch, scale);
  if (cs != LVSA_OK) return cs;
  const size_t bytes = static_cast<size_t>(batch) * T * P * heads * static_cast<size_t>(d) * 2;
  if (!disjoint(out, q, bytes) || !disjoint(out, k, bytes) || !disjoint(out, v, bytes)) return LVSA_ERR_INVALID_ARG;
  if (!ranges_disjoint(out, bytes, lists, static_cast<size_t>(T) * L * 4)) return LVSA_ERR_INVALID_ARG;
  int dev = 0;
  const lvsa_status ds = check_device(&dev);
  if (ds != LVSA_OK) return ds;
  return launch_band(q, k, v, lists, L, T, P, heads, heads, d, batch, scale,
                     one_buffer(out, static_cast<long long>(T) * P, heads), static_cast<cudaStream_t>(stream), dev);
}

extern "C" lvsa_status lvsa_attention_joint(const void* q, const void* k, const void* v, const int32_t* lists, int L,
                                            int T, int tokens_per_frame, int text_tokens, int heads, int d,
                                            int batch, float scale, void* out, void* stream) {
  using namespace lvsa;
  const int P = tokens_per_frame;
  if (!q || !k || !v || !lists || !out) return LVSA_ERR_INVALID_ARG;
  if (T < 1 || P < 1 || heads < 1 || batch < 1 || L < 1 || L > T || text_tokens < 0) return LVSA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return LVSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lists) & 3u))
    return LVSA_ERR_INVALID_ARG;
  const lvsa_status cs = check_sizes(L, T, P, heads, d, batch, scale, text_tokens);
  if (cs != LVSA_OK) return cs;
  const long long tokens = static_cast<long long>(T) * P + text_tokens;
  const size_t bytes = static_cast<size_t>(batch) * tokens * heads * static_cast<size_t>(d) * 2;
  if (!disjoint(out, q, bytes) || !disjoint(out, k, bytes) || !disjoint(out, v, bytes)) return LVSA_ERR_INVALID_ARG;
  if (!ranges_disjoint(out, bytes, lists, static_cast<size_t>(T) * L * 4)) return LVSA_ERR_INVALID_ARG;
  int dev = 0;
  const lvsa_status ds = check_device(&dev);
  if (ds != LVSA_OK) return ds;
  return launch_band(q, k, v, lists, L, T, P, heads, heads, d, batch, scale, one_buffer(out, tokens, heads),
                     static_cast<cudaStream_t>(stream), dev, text_tokens);
}

extern "C" lvsa_status lvsa_attention_to_chunks(const void* q, const void* k, const void* v, const int32_t* lists,
                                                int L, int T, int tokens_per_frame, int heads, int d, int batch,
                                                float scale, void* const* out_chunks, const int* chunk_tokens,
                                                int nchunks, int out_heads, int head0, void* stream) {
  using namespace lvsa;
  const int P = tokens_per_frame;
  if (!q || !k || !v || !lists || !out_chunks || !chunk_tokens) return LVSA_ERR_INVALID_ARG;
  if (T < 1 || P < 1 || heads < 1 || batch < 1 || L < 1 || L > T) return LVSA_ERR_INVALID_ARG;
  if (nchunks < 1 || nchunks > kMaxChunks) return LVSA_ERR_INVALID_ARG;
  if (head0 < 0 || out_heads < 1 || head0 + heads > out_heads || out_heads > 65535) return LVSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(lists) & 3u))
    return LVSA_ERR_INVALID_ARG;
  const lvsa_status cs = check_sizes(L, T, P, heads, d, batch, scale);
  if (cs != LVSA_OK) return cs;
  Route route;
  route.nchunks = nchunks;
  route.head_stride = out_heads;
  route.head0 = head0;
  long long tokens = 0;
  for (int c = 0; c < nchunks; ++c) {
    if (chunk_tokens[c] < 0) return LVSA_ERR_INVALID_ARG;
    route.start[c] = static_cast<int>(tokens);
    tokens += chunk_tokens[c];
    if (tokens > static_cast<long long>(T) * P) return LVSA_ERR_INVALID_ARG;
    route.out[c] = out_chunks[c];
    if (chunk_tokens[c] > 0 && (!out_chunks[c] || !aligned16(out_chunks[c]))) return LVSA_ERR_INVALID_ARG;
  }
  if (tokens != static_cast<long long>(T) * P) return LVSA_ERR_INVALID_ARG;
  route.start[nchunks] = static_cast<int>(tokens);
  // output buffers disjoint from each other, from q, k, v and from the lists: checked on the caller's
  // addresses here (no CUDA call), and again below on the device addresses CUDA reports for them
  auto overlaps = [&](void* const* outs) {
    const size_t in_bytes = static_cast<size_t>(batch) * T * P * heads * static_cast<size_t>(d) * 2;
    const size_t list_bytes = static_cast<size_t>(T) * L * 4;
    for (int c = 0; c < nchunks; ++c) {
      if (chunk_tokens[c] == 0) continue;
      const size_t cb = static_cast<size_t>(batch) * chunk_tokens[c] * out_heads * static_cast<size_t>(d) * 2;
      for (const void* in : {q, k, v})
        if (!ranges_disjoint(outs[c], cb, in, in_bytes)) return true;
      if (!ranges_disjoint(outs[c], cb, lists, list_bytes)) return true;
      for (int e = 0; e < c; ++e) {
        const size_t eb = static_cast<size_t>(batch) * chunk_tokens[e] * out_heads * static_cast<size_t>(d) * 2;
        if (!ranges_disjoint(outs[c], cb, outs[e], eb)) return true;
      }
    }
    return false;
  };
  if (overlaps(out_chunks)) return LVSA_ERR_INVALID_ARG;
  int dev = 0;
  const lvsa_status ds = check_device(&dev);
  if (ds != LVSA_OK) return ds;
  // every buffer must be addressable from this GPU: its own memory, another GPU's with peer access, or
  // mapped (pinned) host memory, written through the device address CUDA reports for it.  A buffer that is
  // not this GPU's memory has its stores released at system scope.
  const PeerOps ops = runtime_peer_ops();
  for (int c = 0; c < nchunks; ++c) {
    if (chunk_tokens[c] == 0) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, out_chunks[c]) != cudaSuccess) {
      (void)cudaGetLastError();
      return LVSA_ERR_INVALID_ARG;
    }
    void* dptr = nullptr;
    int remote = 0;
    const lvsa_status as = device_address(at, dev, ops, &dptr, &remote);
    if (as != LVSA_OK) return as;
    if (!aligned16(dptr)) return LVSA_ERR_INVALID_ARG;
    route.out[c] = dptr;
    route.routed |= remote;
  }
  if (overlaps(route.out)) return LVSA_ERR_INVALID_ARG;
  return launch_band(q, k, v, lists, L, T, P, heads, heads, d, batch, scale, route, static_cast<cudaStream_t>(stream),
                     dev);
}

extern "C" lvsa_status lvsa_attention_host(const void* q_host, const void* k_host, const void* v_host,
                                           const int32_t* lists_host, int L, int T, int tokens_per_frame, int heads,
                                           int d, int batch, float scale, void* out_host, void* q_dev, void* k_dev,
                                           void* v_dev, int32_t* lists_dev, void* out_dev, int heads_per_band,
                                           void* stream) {
  using namespace lvsa;
  const int P = tokens_per_frame;
  if (!q_host || !k_host || !v_host || !lists_host || !out_host) return LVSA_ERR_INVALID_ARG;
  if (!q_dev || !k_dev || !v_dev || !lists_dev || !out_dev) return LVSA_ERR_INVALID_ARG;
  if (T < 1 || P < 1 || heads < 1 || batch < 1 || L < 1 || L > T) return LVSA_ERR_INVALID_ARG;
  if (heads_per_band < 0 || heads_per_band > heads) return LVSA_ERR_INVALID_ARG;
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || !aligned16(out_dev) ||
      (reinterpret_cast<uintptr_t>(lists_dev) & 3u))
    return LVSA_ERR_INVALID_ARG;
  const lvsa_status cs = check_sizes(L, T, P, heads, d, batch, scale);
  if (cs != LVSA_OK) return cs;
  const size_t row_bytes = static_cast<size_t>(heads) * d * 2;
  const size_t rows = static_cast<size_t>(batch) * T * P;
  const size_t bytes = rows * row_bytes;
  if (!disjoint(out_dev, q_dev, bytes) || !disjoint(out_dev, k_dev, bytes) || !disjoint(out_dev, v_dev, bytes))
    return LVSA_ERR_INVALID_ARG;
  if (!disjoint(out_host, q_host, bytes) || !disjoint(out_host, k_host, bytes) || !disjoint(out_host, v_host, bytes))
    return LVSA_ERR_INVALID_ARG;
  const size_t list_bytes = static_cast<size_t>(T) * L * 4;
  if (!ranges_disjoint(out_dev, bytes, lists_dev, list_bytes) || !ranges_disjoint(out_host, bytes, lists_host, list_bytes))
    return LVSA_ERR_INVALID_ARG;
  int dev = 0;
  const lvsa_status ds = check_device(&dev);
  if (ds != LVSA_OK) return ds;
  // default: one head per band, so that only one head's upload (before the first kernel) and one
  // head's readback (after the last) are not hidden; a band of one head still fills the GPU at
  // video sizes (T*P/256 query blocks per batch entry)
  const int hb = heads_per_band > 0 ? heads_per_band : 1;
  const int bands = (heads + hb - 1) / hb;
  // The first band's Q is uploaded, and the last band's output read back, in pieces of whole query blocks,
  // each piece's kernel launched (or its rows read back) as soon as it can: only a quarter of a band's Q
  // upload precedes the first kernel, and only a quarter of a band's readback follows the last one.
  // (Batch 1 and frames of at least 256 tokens, where a piece of query blocks is one range of rows.)
  constexpr int kPieces = 4;
  const Blocks bl = query_blocks(T, P, 0);
  const bool pieces = batch == 1 && bl.straddle && bl.nvblocks >= 2 * kPieces;
  std::lock_guard<std::mutex> g(g_pipe_mu);
  NvtxRange whole("lvsa_attention_host");
  HostPipe* hp = nullptr;
  lvsa_status r = pipe_for(dev, bands + 2 * kPieces, &hp);  // at most 2 bands go in pieces
  if (r != LVSA_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int next_ev = 0;
  auto event = [&]() { return hp->ev[next_ev++]; };
  cudaEvent_t ev_start = event(), ev_done = event();
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // the copies into the staging buffers wait for earlier work on the caller's stream
  if (!ok(cudaEventRecord(ev_start, st)) || !ok(cudaStreamWaitEvent(hp->h2d, ev_start, 0)) ||
      !ok(cudaStreamWaitEvent(hp->d2h, ev_start, 0)))
    return LVSA_ERR_CUDA;
  if (!ok(cudaMemcpyAsync(lists_dev, lists_host, static_cast<size_t>(T) * L * 4, cudaMemcpyHostToDevice, hp->h2d)))
    return LVSA_ERR_CUDA;
  const char* src[3] = {static_cast<const char*>(q_host), static_cast<const char*>(k_host),
                        static_cast<const char*>(v_host)};
  char* dst[3] = {static_cast<char*>(q_dev), static_cast<char*>(k_dev), static_cast<char*>(v_dev)};
  const long long tokens = static_cast<long long>(T) * P;
  constexpr int kRows = kQTiles * kBM;
  for (int gi = 0; gi < bands; ++gi) {
    const int h0 = gi * hb;
    const int hn = std::min(hb, heads - h0);
    const size_t off = static_cast<size_t>(h0) * d * 2;
    const size_t width = static_cast<size_t>(hn) * d * 2;
    const bool q_in_pieces = pieces && gi == 0;
    const bool out_in_pieces = pieces && gi == bands - 1;
    const int npieces = (q_in_pieces || out_in_pieces) ? kPieces : 1;
    // band gi of K, V (and Q, unless it goes up in pieces): a column band of every token row
    {
      NvtxRange r("lvsa.upload band", gi);
      for (int t = q_in_pieces ? 1 : 0; t < 3; ++t)
        if (!ok(cudaMemcpy2DAsync(dst[t] + off, row_bytes, src[t] + off, row_bytes, width, rows,
                                  cudaMemcpyHostToDevice, hp->h2d)))
          return LVSA_ERR_CUDA;
    }
    for (int c = 0; c < npieces; ++c) {
      // query blocks [b0, b1) = rows [b0 * 256, b1 * 256) of the sequence
      const long long b0 = npieces == 1 ? 0 : bl.nvblocks * c / npieces;
      const long long b1 = npieces == 1 ? bl.nvblocks : bl.nvblocks * (c + 1) / npieces;
      const size_t row0 = static_cast<size_t>(b0) * kRows;
      const size_t nrows = static_cast<size_t>(std::min(b1 * kRows, tokens)) - row0;
      if (q_in_pieces &&
          !ok(cudaMemcpy2DAsync(dst[0] + row0 * row_bytes + off, row_bytes, src[0] + row0 * row_bytes + off, row_bytes,
                                width, nrows, cudaMemcpyHostToDevice, hp->h2d)))
        return LVSA_ERR_CUDA;
      NvtxRange kr("lvsa.kernel band", gi);
      cudaEvent_t ev_in = event(), ev_k = event();
      cudaStream_t ks = hp->k[(gi + c) & 1];
      if (!ok(cudaEventRecord(ev_in, hp->h2d)) || !ok(cudaStreamWaitEvent(ks, ev_in, 0))) return LVSA_ERR_CUDA;
      r = launch_band(dst[0] + off, dst[1] + off, dst[2] + off, lists_dev, L, T, P, hn, heads, d, batch, scale,
                      one_buffer(static_cast<char*>(out_dev) + off, tokens, heads), ks, dev, 0,
                      npieces == 1 ? 0 : static_cast<int>(b0), npieces == 1 ? -1 : static_cast<int>(b1 - b0));
      if (r != LVSA_OK) return r;
      if (!ok(cudaEventRecord(ev_k, ks)) || !ok(cudaStreamWaitEvent(hp->d2h, ev_k, 0))) return LVSA_ERR_CUDA;
      if (out_in_pieces &&
          !ok(cudaMemcpy2DAsync(static_cast<char*>(out_host) + row0 * row_bytes + off, row_bytes,
                                static_cast<const char*>(out_dev) + row0 * row_bytes + off, row_bytes, width, nrows,
                                cudaMemcpyDeviceToHost, hp->d2h)))
        return LVSA_ERR_CUDA;
    }
    // the whole band's output, once every piece's kernel is done
    NvtxRange rr("lvsa.readback band", gi);
    if (!out_in_pieces &&
        !ok(cudaMemcpy2DAsync(static_cast<char*>(out_host) + off, row_bytes, static_cast<const char*>(out_dev) + off,
                              row_bytes, width, rows, cudaMemcpyDeviceToHost, hp->d2h)))
      return LVSA_ERR_CUDA;
  }
  // later work on the caller's stream sees the whole output in host memory (every band's readback
  // waited for its kernel, so this also orders every kernel before that work)
  if (!ok(cudaEventRecord(ev_done, hp->d2h)) || !ok(cudaStreamWaitEvent(st, ev_done, 0))) return LVSA_ERR_CUDA;
  return LVSA_OK;
}

// ------------------------------------------------------------------ staging without allocation
// lvsa_attention_host_static stages its inputs and output in this array instead of caller buffers or
// allocations.  In host code `g_static_scratch` names a host-side stand-in, not device memory: the device
// address is looked up once per device with cudaGetSymbolAddress (that device current) and kept.
namespace lvsa {
namespace {
constexpr size_t kStaticScratchBytes = LVSA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_base[64] = {};

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// The array's device address on device `dev` (the current device); null if CUDA cannot give it.
void* static_scratch(int dev) {
  std::lock_guard<std::mutex> g(g_static_mu);
  if (!g_static_base[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    g_static_base[dev] = ptr;
  }
  return g_static_base[dev];
}
}  // namespace
}  // namespace lvsa

extern "C" lvsa_status lvsa_attention_host_static(const void* q_host, const void* k_host, const void* v_host,
                                                  const int32_t* lists_host, int L, int T, int tokens_per_frame,
                                                  int heads, int d, int batch, float scale, void* out_host,
                                                  void* stream) {
  using namespace lvsa;
  const int P = tokens_per_frame;
  if (!q_host || !k_host || !v_host || !lists_host || !out_host) return LVSA_ERR_INVALID_ARG;
  if (T < 1 || P < 1 || heads < 1 || batch < 1 || L < 1 || L > T) return LVSA_ERR_INVALID_ARG;
  const lvsa_status cs = check_sizes(L, T, P, heads, d, batch, scale);
  if (cs != LVSA_OK) return cs;
  const size_t bytes = static_cast<size_t>(batch) * T * P * heads * static_cast<size_t>(d) * 2;
  const size_t list_bytes = static_cast<size_t>(T) * L * 4;
  if (!disjoint(out_host, q_host, bytes) || !disjoint(out_host, k_host, bytes) || !disjoint(out_host, v_host, bytes) ||
      !ranges_disjoint(out_host, bytes, lists_host, list_bytes))
    return LVSA_ERR_INVALID_ARG;
  // layout in the array: Q, K, V, output, lists, each at a 256-byte boundary
  const size_t slot = round256(bytes);
  if (slot > kStaticScratchBytes / 4 || 4 * slot + round256(list_bytes) > kStaticScratchBytes)
    return LVSA_ERR_INVALID_ARG;
  int dev = 0;
  const lvsa_status ds = check_device(&dev);
  if (ds != LVSA_OK) return ds;
  if (dev >= 64) return LVSA_ERR_UNSUPPORTED;
  char* base = static_cast<char*>(static_scratch(dev));
  if (!base) return LVSA_ERR_CUDA;
  char* q_d = base;
  char* k_d = base + slot;
  char* v_d = base + 2 * slot;
  char* out_d = base + 3 * slot;
  int32_t* lists_d = reinterpret_cast<int32_t*>(base + 4 * slot);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const struct { void* dst; const void* src; size_t n; } up[4] = {
      {lists_d, lists_host, list_bytes}, {q_d, q_host, bytes}, {k_d, k_host, bytes}, {v_d, v_host, bytes}};
  for (const auto& c : up)
    if (cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, st) != cudaSuccess) return LVSA_ERR_CUDA;
  const lvsa_status r = launch_band(q_d, k_d, v_d, lists_d, L, T, P, heads, heads, d, batch, scale,
                                    one_buffer(out_d, static_cast<long long>(T) * P, heads), st, dev);
  if (r != LVSA_OK) return r;
  if (cudaMemcpyAsync(out_host, out_d, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return LVSA_ERR_CUDA;
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_get_device_status(unsigned int* flags, int clear) {
  if (!flags) return LVSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return LVSA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_lvsa_dev_status, sizeof(v)) != cudaSuccess) return LVSA_ERR_CUDA;
  *flags = v;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_lvsa_dev_status, &zero, sizeof(zero)) != cudaSuccess) return LVSA_ERR_CUDA;
  }
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_set_wait_budget_ns(unsigned long long ns) {
  if (ns > lvsa::kMaxWaitBudgetNs) return LVSA_ERR_INVALID_ARG;
  lvsa::g_wait_ns = ns < lvsa::kMinWaitBudgetNs ? lvsa::kMinWaitBudgetNs : ns;
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_watchdog_selftest(unsigned long long budget_ns, void* stream) {
  if (budget_ns < 1000ull) budget_ns = 1000ull;
  if (budget_ns > 10000000000ull) return LVSA_ERR_INVALID_ARG;
  lvsa::watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(lvsa::wait_budget_cycles(budget_ns));
  return cudaGetLastError() == cudaSuccess ? LVSA_OK : LVSA_ERR_CUDA;
}

extern "C" const char* lvsa_status_string(int status) {
  switch (status) {
    case LVSA_OK: return "LVSA_OK";
    case LVSA_ERR_INVALID_ARG: return "LVSA_ERR_INVALID_ARG";
    case LVSA_ERR_UNSUPPORTED: return "LVSA_ERR_UNSUPPORTED";
    case LVSA_ERR_CUDA: return "LVSA_ERR_CUDA";
    case LVSA_ERR_TIMEOUT: return "LVSA_ERR_TIMEOUT";
    case LVSA_ERR_BUFFER_TOO_SMALL: return "LVSA_ERR_BUFFER_TOO_SMALL";
    case LVSA_ERR_BAD_LIST: return "LVSA_ERR_BAD_LIST";
    default: return "LVSA_ERR_UNKNOWN";
  }
}

extern "C" int lvsa_version(void) { return 100; }
