// Sequence-parallel exchange of the LVSA attention path: the DeepSpeed-Ulysses layout under which the
// method runs Wan 2.2-A14B on 8 NPUs (techwalker article "华为巴黎研究院让AI视频“不再原地打转”",
// section 五).  Each rank holds a token range of Q, K and V for every head and computes attention for a
// band of heads over the whole sequence; heads are independent because A(t) is shared by every head.
//
//   lvsa_seq_to_heads   gathers this rank's band of heads from every rank's token range into one local
//                       [batch][tokens][band][d] buffer per tensor, by plain 16-byte loads from the other
//                       GPUs' memory (NVLink peer mappings): the sequence-to-head all-to-all as one kernel.
//   lvsa_ipc_*          export a device buffer as a CUDA IPC handle and map another process's buffer into
//                       this one, so the gather and the attention epilogue can address peers directly.
//
// The attention call that stores each output row into the buffer of the rank owning its token
// (lvsa_attention_to_chunks) is in attention.cu.  Nothing here waits on another GPU: the caller orders
// the ranks (a process-group barrier before the gather and after the attention).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <array>
#include <climits>
#include <cstring>
#include <map>
#include <mutex>

#include "buffer_checks.h"
#include "lvsa.h"

namespace lvsa {
namespace {

constexpr int kMaxExchangeChunks = 64;
constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;

struct GatherParams {
  const uint4* src[3][kMaxExchangeChunks];  // q, k, v token ranges: [batch][tokens of c][heads][d]
  uint4* dst[3];                            // [batch][tokens][band][d]
  int start[kMaxExchangeChunks + 1];        // range c holds tokens [start[c], start[c + 1])
  int tokens;                               // start[nchunks]
  int vec_src;                              // 16-byte vectors per source token row (heads * d / 8)
  int vec_band;                             // 16-byte vectors per band row (band * d / 8)
  int vec_head0;                            // first vector of the band within a source row
};

// grid (x: row groups, y: source range c, z: tensor + 3 * batch entry); block (vx, ry): vx vectors of a
// row by ry rows.  Each thread copies kGatherUnroll rows per round, loads first, so that several
// peer reads are in flight per thread.
__global__ void __launch_bounds__(kGatherThreads) seq_to_heads_kernel(const __grid_constant__ GatherParams p) {
  const int c = blockIdx.y;
  const int x = blockIdx.z % 3;
  const int b = blockIdx.z / 3;
  const int c0 = p.start[c];
  const int rows = p.start[c + 1] - c0;
  if (rows <= 0) return;
  const uint4* src = p.src[x][c] + static_cast<size_t>(b) * rows * p.vec_src + p.vec_head0;
  uint4* dst = p.dst[x] + (static_cast<size_t>(b) * p.tokens + c0) * p.vec_band;
  const int ry = blockDim.y;
  const int stride = gridDim.x * ry;
  for (int r = blockIdx.x * ry + threadIdx.y; r < rows; r += kGatherUnroll * stride) {
    for (int v = threadIdx.x; v < p.vec_band; v += blockDim.x) {
      uint4 buf[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int rr = r + u * stride;
        if (rr < rows) buf[u] = src[static_cast<size_t>(rr) * p.vec_src + v];
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int rr = r + u * stride;
        if (rr < rows) dst[static_cast<size_t>(rr) * p.vec_band + v] = buf[u];
      }
    }
  }
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool disjoint(const void* a, size_t abytes, const void* b, size_t bbytes) { return ranges_disjoint(a, abytes, b, bbytes); }

// ------------------------------------------------------------------ IPC mappings
using AddrRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

AddrRangeFn addr_range_fn() {
  static AddrRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddrRangeFn>(ptr);
  });
  return fn;
}

// One mapping per (device, exporting allocation); several imported pointers may share it.
struct Mapping {
  void* base = nullptr;
  int refs = 0;
};
using HandleKey = std::array<unsigned char, sizeof(cudaIpcMemHandle_t) + sizeof(int)>;
std::mutex g_ipc_mu;
std::map<HandleKey, Mapping> g_maps;
std::map<void*, std::pair<HandleKey, int>> g_imported;  // pointer handed out -> (mapping, times handed out)

}  // namespace
}  // namespace lvsa

extern "C" lvsa_status lvsa_seq_to_heads(const void* const* q_chunks, const void* const* k_chunks,
                                         const void* const* v_chunks, const int* chunk_tokens, int nchunks,
                                         int heads, int head0, int band, int d, int batch, void* q_band,
                                         void* k_band, void* v_band, void* stream) {
  using namespace lvsa;
  if (!q_chunks || !k_chunks || !v_chunks || !chunk_tokens || !q_band || !k_band || !v_band)
    return LVSA_ERR_INVALID_ARG;
  if (nchunks < 1 || nchunks > kMaxExchangeChunks) return LVSA_ERR_INVALID_ARG;
  if (heads < 1 || band < 1 || head0 < 0 || head0 + band > heads || batch < 1 || batch > 21845)
    return LVSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LVSA_ERR_UNSUPPORTED;
  GatherParams gp;
  const void* const* tables[3] = {q_chunks, k_chunks, v_chunks};
  void* dsts[3] = {q_band, k_band, v_band};
  long long tokens = 0;
  int max_rows = 0;
  gp.start[0] = 0;
  for (int c = 0; c < nchunks; ++c) {
    if (chunk_tokens[c] < 0) return LVSA_ERR_INVALID_ARG;
    tokens += chunk_tokens[c];
    if (tokens > INT_MAX) return LVSA_ERR_INVALID_ARG;
    gp.start[c + 1] = static_cast<int>(tokens);
    max_rows = chunk_tokens[c] > max_rows ? chunk_tokens[c] : max_rows;
    for (int x = 0; x < 3; ++x) {
      const void* s = tables[x][c];
      if (chunk_tokens[c] > 0 && (!s || !aligned16(s))) return LVSA_ERR_INVALID_ARG;
      gp.src[x][c] = static_cast<const uint4*>(s);
    }
  }
  for (int c = nchunks + 1; c <= kMaxExchangeChunks; ++c) gp.start[c] = static_cast<int>(tokens);
  for (int c = nchunks; c < kMaxExchangeChunks; ++c)
    for (int x = 0; x < 3; ++x) gp.src[x][c] = nullptr;
  if (tokens < 1) return LVSA_ERR_INVALID_ARG;
  const size_t band_bytes = static_cast<size_t>(batch) * tokens * band * d * 2;
  for (int x = 0; x < 3; ++x) {
    if (!aligned16(dsts[x])) return LVSA_ERR_INVALID_ARG;
    gp.dst[x] = static_cast<uint4*>(dsts[x]);
    for (int y = 0; y < x; ++y)
      if (!disjoint(dsts[x], band_bytes, dsts[y], band_bytes)) return LVSA_ERR_INVALID_ARG;
    // a band buffer may not overlap a source range (local ones can be checked; a peer mapping has its own
    // addresses, so it never overlaps a local buffer)
    for (int c = 0; c < nchunks; ++c) {
      const size_t cb = static_cast<size_t>(batch) * chunk_tokens[c] * heads * d * 2;
      for (int y = 0; y < 3; ++y)
        if (chunk_tokens[c] > 0 && !disjoint(dsts[x], band_bytes, tables[y][c], cb)) return LVSA_ERR_INVALID_ARG;
    }
  }
  gp.tokens = static_cast<int>(tokens);
  gp.vec_src = heads * d / 8;
  gp.vec_band = band * d / 8;
  gp.vec_head0 = head0 * d / 8;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LVSA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LVSA_ERR_CUDA;
  // every source range must be addressable from this GPU (its memory, a peer's with peer access, or mapped
  // host memory); the kernel loads through the device address CUDA reports for it
  const PeerOps ops{cudaDeviceCanAccessPeer, cudaDeviceEnablePeerAccess, cudaGetLastError};
  for (int c = 0; c < nchunks; ++c) {
    if (chunk_tokens[c] == 0) continue;
    for (int x = 0; x < 3; ++x) {
      cudaPointerAttributes at;
      if (cudaPointerGetAttributes(&at, tables[x][c]) != cudaSuccess) {
        (void)cudaGetLastError();
        return LVSA_ERR_INVALID_ARG;
      }
      void* dptr = nullptr;
      int remote = 0;
      const lvsa_status as = device_address(at, dev, ops, &dptr, &remote);
      if (as != LVSA_OK) return as;
      if (!aligned16(dptr)) return LVSA_ERR_INVALID_ARG;
      gp.src[x][c] = static_cast<const uint4*>(dptr);
    }
  }
  const int vx = gp.vec_band < kGatherThreads ? gp.vec_band : kGatherThreads;
  const int ry = kGatherThreads / vx;
  // about 8 CTAs of 256 threads per SM over the whole launch, at least one per source range
  const long long per_range = (8LL * sms + 3LL * batch * nchunks - 1) / (3LL * batch * nchunks);
  const long long need = (static_cast<long long>(max_rows) + ry - 1) / ry;
  const long long gx = need < per_range ? need : per_range;
  dim3 grid(static_cast<unsigned>(gx > 0 ? gx : 1), static_cast<unsigned>(nchunks), static_cast<unsigned>(3 * batch));
  seq_to_heads_kernel<<<grid, dim3(vx, ry), 0, static_cast<cudaStream_t>(stream)>>>(gp);
  return cudaGetLastError() == cudaSuccess ? LVSA_OK : LVSA_ERR_CUDA;
}

extern "C" lvsa_status lvsa_ipc_export(const void* dev_ptr, void* handle) {
  using namespace lvsa;
  if (!dev_ptr || !handle) return LVSA_ERR_INVALID_ARG;
  auto range = addr_range_fn();
  if (!range) return LVSA_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return LVSA_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return LVSA_ERR_CUDA;
  const uint64_t offset = reinterpret_cast<uintptr_t>(dev_ptr) - static_cast<uintptr_t>(base);
  unsigned char* out = static_cast<unsigned char*>(handle);
  std::memcpy(out, &h, sizeof(h));
  std::memcpy(out + sizeof(h), &offset, sizeof(offset));
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_ipc_import(const void* handle, void** dev_ptr) {
  using namespace lvsa;
  if (!handle || !dev_ptr) return LVSA_ERR_INVALID_ARG;
  *dev_ptr = nullptr;
  cudaIpcMemHandle_t h;
  uint64_t offset = 0;
  std::memcpy(&h, handle, sizeof(h));
  std::memcpy(&offset, static_cast<const unsigned char*>(handle) + sizeof(h), sizeof(offset));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LVSA_ERR_CUDA;
  HandleKey key;
  std::memcpy(key.data(), &h, sizeof(h));
  std::memcpy(key.data() + sizeof(h), &dev, sizeof(dev));
  std::lock_guard<std::mutex> g(g_ipc_mu);
  Mapping& m = g_maps[key];
  if (!m.base) {
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
      g_maps.erase(key);
      return LVSA_ERR_CUDA;
    }
    m.base = base;
  }
  ++m.refs;
  void* p = static_cast<char*>(m.base) + offset;
  auto& rec = g_imported[p];
  rec.first = key;
  ++rec.second;
  *dev_ptr = p;
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_ipc_release(void* dev_ptr) {
  using namespace lvsa;
  if (!dev_ptr) return LVSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(g_ipc_mu);
  auto it = g_imported.find(dev_ptr);
  if (it == g_imported.end()) return LVSA_ERR_INVALID_ARG;
  const HandleKey key = it->second.first;
  if (--it->second.second == 0) g_imported.erase(it);
  auto mit = g_maps.find(key);
  if (mit == g_maps.end()) return LVSA_ERR_INVALID_ARG;
  if (--mit->second.refs == 0) {
    const cudaError_t e = cudaIpcCloseMemHandle(mit->second.base);
    g_maps.erase(mit);
    if (e != cudaSuccess) return LVSA_ERR_CUDA;
  }
  return LVSA_OK;
}
