// LVSA frame-granular block-sparse attention for B200 (sm_100a).
//
// "LVSA: Training-Free Sparse Attention for Long Video Diffusion" (gist.science
// technical summary, section 2 "Core Mechanism" and "Complexity"): a query token
// of frame t attends only to the tokens of the frames in A(t); one softmax over
// all of them; cost O(T * C * P^2 * d).
//
// Kernel structure (one CTA per (query frame t, 128-row query tile, head, batch)):
//   warp 4      TMA producer: Q tile once, then K/V tiles of the listed frames
//               into a ring of shared-memory slots.  The frame list is walked as
//               runs of consecutive frames; a run is one contiguous token range,
//               cut into 128-token tiles (the last one partial).  The gather is
//               done by TMA coordinates: no mask is ever materialised.
//   warp 5      TMEM allocator and single-thread tcgen05.mma issuer:
//                 S(j) = Q K_j^T  into one of two TMEM S buffers (SS form)
//                 O   += P(j) V_j with P read from TMEM (TS form)
//               A partial tile issues N (QK) and K (PV) rounded up to 16 only.
//   warps 0-3   softmax, one thread per query row (TMEM lane): online softmax in
//               the exp2 domain with a lazily updated running max (O in TMEM is
//               rescaled only when the max grows by more than 2^8), P written
//               back into the S buffer as bf16, epilogue O / l -> bf16 -> HBM.
// Every wait is bounded: when its time budget runs out the CTA stops, sets a
// device status bit, lets its in-flight copies and MMAs finish and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <climits>
#include <cmath>
#include <mutex>

#include "lvsa.h"
#include "sm100.cuh"

__device__ unsigned int g_lvsa_dev_status = 0;

namespace lvsa {
using namespace sm100;

constexpr int kBM = 128;          // query rows per tile = MMA M
constexpr int kBN = 128;          // keys per K/V tile = largest MMA N of QK^T
constexpr int kThreads = 192;     // 4 softmax warps + TMA warp + MMA warp
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kTmemCols = 512;
constexpr int kSCol0 = 0;         // S/P buffer 0: TMEM columns [0,128)
constexpr int kSCol1 = 128;       // S/P buffer 1: TMEM columns [128,256)
constexpr int kOCol = 256;        // O accumulator: TMEM columns [256, 256+d)
constexpr int kChunkBytes = kBM * 128;    // one 128-byte-wide swizzle column of a 128-row tile
constexpr float kRescaleLog2 = 8.0f;      // rescale O only when the max grows by > 2^8

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kSlots = (D == 128) ? 5 : 10;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kTileBytes;
  static constexpr int kOffBar = kOffRing + kSlots * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct KernelParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  __nv_bfloat16* out;
  const int32_t* lists;
  int T, P, H, L;
  int qtiles;        // ceil(P / 128)
  float scale_log2;  // softmax scale * log2(e)
  unsigned long long wait_ns;
};

// ------------------------------------------------------------------ bounded waits
struct Watch {
  unsigned long long budget_ns;
  volatile int* abort_flag;  // shared memory, CTA-wide
};

// Returns false when the budget ran out (status bit set) or another role of the
// CTA already gave up.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const Watch& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort_flag) return false;
    if (global_timer_ns() - t0 > w.budget_ns) {
      *w.abort_flag = 1;
      atomicOr(&g_lvsa_dev_status, LVSA_DEV_TIMEOUT);
      return false;
    }
  }
}

// Used only while shutting down after an abort: ignores the abort flag.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, unsigned long long budget_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > budget_ns) {
      atomicOr(&g_lvsa_dev_status, LVSA_DEV_TIMEOUT);
      return;
    }
  }
}

// ------------------------------------------------------------------ K/V tile walk
// Walks the frame list of one query frame as runs of consecutive frames and
// cuts each run's token range into tiles of at most 128 tokens.  Every role
// of the CTA walks the same sequence.
struct TileWalk {
  const int32_t* list;
  int L, T, P;
  int li = 0, pos = 0, end = 0;
  bool bad = false;

  __device__ TileWalk(const int32_t* l, int L_, int T_, int P_) : list(l), L(L_), T(T_), P(P_) {}

  __device__ __forceinline__ bool next(int& tok, int& nvalid) {
    while (pos >= end) {
      if (li >= L) return false;
      const int f0 = __ldg(list + li++);
      if (f0 < 0 || f0 >= T) {
        bad = true;
        continue;
      }
      int f1 = f0;
      while (li < L) {
        const int f = __ldg(list + li);
        if (f != f1 + 1 || f >= T) break;
        f1 = f;
        ++li;
      }
      pos = f0 * P;
      end = (f1 + 1) * P;
    }
    tok = pos;
    nvalid = min(kBN, end - pos);
    pos += nvalid;
    return true;
  }
};

// ------------------------------------------------------------------ the kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1) lvsa_attention_kernel(const __grid_constant__ KernelParams p) {
  using Cf = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Cf::kOffQ;
  uint8_t* sRing = smem + Cf::kOffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kOffBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bar_full + Cf::kSlots;
  uint64_t* bar_s = bar_empty + Cf::kSlots;  // [2] S(j) ready in TMEM
  uint64_t* bar_p = bar_s + 2;               // [2] P(j) written to TMEM (128 arrivals)
  uint64_t* bar_o = bar_p + 2;               // PV(j) finished
  uint64_t* bar_drain = bar_o + 1;           // all MMAs of the CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x % p.qtiles;
  const int t = blockIdx.x / p.qtiles;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int32_t* list = p.lists + static_cast<size_t>(t) * p.L;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < Cf::kSlots; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
    }
    mbar_init(bar_s + 0, 1);
    mbar_init(bar_s + 1, 1);
    mbar_init(bar_p + 0, 4 * 32);
    mbar_init(bar_p + 1, 4 * 32);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watch w{p.wait_ns, abort_flag};

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int col0 = h * D;
      const int qrow = t * p.P + qt * kBM;
      mbar_arrive_expect_tx(bar_q, Cf::kTileBytes);
#pragma unroll
      for (int c = 0; c < Cf::kChunks; ++c) tma_load_3d(sQ + c * kChunkBytes, &p.tm_q, bar_q, col0 + c * 64, qrow, b);

      int issued = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* tm, int tok) {
        const int slot = issued % Cf::kSlots;
        const uint32_t phase = (issued / Cf::kSlots) & 1;
        if (!wait_bounded(bar_empty + slot, phase ^ 1, w)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(bar_full + slot, Cf::kTileBytes);
        uint8_t* dst = sRing + slot * Cf::kTileBytes;
#pragma unroll
        for (int c = 0; c < Cf::kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, tm, bar_full + slot, col0 + c * 64, tok, b);
        ++issued;
      };
      // consumption order of the MMA warp: K0, K1, V0, K2, V1, ..., K(n-1), V(n-2), V(n-1)
      TileWalk walk(list, p.L, p.T, p.P);
      int tok, nv, prev = -1;
      while (ok && walk.next(tok, nv)) {
        load(&p.tm_k, tok);
        if (ok && prev >= 0) load(&p.tm_v, prev);
        prev = tok;
      }
      if (ok && prev >= 0) load(&p.tm_v, prev);
      if (walk.bad) atomicOr(&g_lvsa_dev_status, LVSA_DEV_BAD_LIST);
      if (!ok) {
        // stopped early: let every copy still in flight land before the CTA exits
        wait_drain(bar_q, 0, p.wait_ns);
        const int first = issued > Cf::kSlots ? issued - Cf::kSlots : 0;
        for (int i = first; i < issued; ++i) wait_drain(bar_full + i % Cf::kSlots, (i / Cf::kSlots) & 1, p.wait_ns);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sq = smem_u32(sQ);
      const uint32_t sr = smem_u32(sRing);
      const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      int consumed = 0;
      bool ok = wait_bounded(bar_q, 0, w);
      auto issue_pv = [&](int i, int n_mma) {
        const int slot = consumed % Cf::kSlots;
        const uint32_t phase = (consumed / Cf::kSlots) & 1;
        if (!wait_bounded(bar_p + (i & 1), (i >> 1) & 1, w) || !wait_bounded(bar_full + slot, phase, w)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t v_addr = sr + slot * Cf::kTileBytes;
        const uint32_t p_tmem = tmem + ((i & 1) ? kSCol1 : kSCol0);
        for (int kk = 0; kk < n_mma / 16; ++kk) {
          // B = V tile, MN-major (d contiguous): 64-wide d chunks 16 KB apart (LBO), 8-key groups 1 KB apart (SBO)
          const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 16 * 128, kChunkBytes, 1024);
          mma_ts(tmem + kOCol, p_tmem + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_empty + slot);
        mma_commit(bar_o);
        ++consumed;
      };
      TileWalk walk(list, p.L, p.T, p.P);
      int tok, nv, j = 0, prev_n = 0;
      while (ok && walk.next(tok, nv)) {
        const int n_mma = (nv + 15) & ~15;
        const int slot = consumed % Cf::kSlots;
        const uint32_t phase = (consumed / Cf::kSlots) & 1;
        if (!wait_bounded(bar_full + slot, phase, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = sr + slot * Cf::kTileBytes;
        const uint32_t idesc_qk = idesc_bf16_f32(kBM, n_mma, false);
        const uint32_t s_tmem = tmem + ((j & 1) ? kSCol1 : kSCol0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // A = Q, B = K, both K-major: 16-element (32-byte) steps inside a 128-byte swizzle row
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          mma_ss(s_tmem, smem_desc_sw128(sq + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_empty + slot);
        mma_commit(bar_s + (j & 1));
        ++consumed;
        if (j > 0) issue_pv(j - 1, prev_n);
        prev_n = n_mma;
        ++j;
      }
      if (ok && j > 0) issue_pv(j - 1, prev_n);
      // every MMA issued must be complete before TMEM is released
      mma_commit(bar_drain);
      wait_drain(bar_drain, 0, p.wait_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
    const int r = threadIdx.x;  // query row of the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_tmem = tmem + lane_off + kOCol;
    const float sl2 = p.scale_log2;
    float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale by < 8)
    float l = 0.f;        // running sum of exp2(scaled s - m)
    bool ok = true;
    int j = 0;
    TileWalk walk(list, p.L, p.T, p.P);
    int tok, nv;
    while (walk.next(tok, nv)) {
      const uint32_t s_tmem = tmem + lane_off + ((j & 1) ? kSCol1 : kSCol0);
      ok = __all_sync(0xffffffffu, wait_bounded(bar_s + (j & 1), (j >> 1) & 1, w));
      if (!ok) break;
      tc_fence_after();
      float s[kBN];
      tmem_ld32(s_tmem + 0, s + 0);
      if (nv > 32) tmem_ld32(s_tmem + 32, s + 32);
      if (nv > 64) tmem_ld32(s_tmem + 64, s + 64);
      if (nv > 96) tmem_ld32(s_tmem + 96, s + 96);
      tmem_wait_ld_regs(s + 0);
      tmem_wait_ld_regs(s + 32);
      tmem_wait_ld_regs(s + 64);
      tmem_wait_ld_regs(s + 96);
      if (nv < kBN) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i >= nv) s[i] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = s[u];
#pragma unroll
      for (int i = 8; i < kBN; ++i) mx[i & 7] = fmaxf(mx[i & 7], s[i]);
      const float tile_max = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
      float alpha = 1.f;
      if (tile_max > m + kRescaleLog2) {
        alpha = ex2(m - tile_max);
        l *= alpha;
        m = tile_max;
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O holds PV(0..j-1): wait for PV(j-1), then rescale this thread's row
        ok = __all_sync(0xffffffffu, wait_bounded(bar_o, (j - 1) & 1, w));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(o_tmem + 32 * c, o);
          tmem_wait_ld_regs(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(o_tmem + 32 * c, o);
        }
      }
      const float neg_m = -m;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c == 0 || nv > 32 * c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float e0 = ex2(fmaf(s[32 * c + 2 * i], sl2, neg_m));
            const float e1 = ex2(fmaf(s[32 * c + 2 * i + 1], sl2, neg_m));
            ls[i & 3] += e0 + e1;
            pk[i] = pack_bf16x2(e0, e1);
          }
          tmem_st16(s_tmem + 16 * c, pk);  // P overwrites the first half of the S buffer
        }
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p + (j & 1));
      ++j;
    }
    if (ok && j > 0) {
      ok = __all_sync(0xffffffffu, wait_bounded(bar_o, (j - 1) & 1, w));
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.f / l;
        const int row = qt * kBM + r;
        const bool valid = row < p.P;
        const size_t ltok = static_cast<size_t>(p.T) * p.P;
        __nv_bfloat16* dst =
            p.out + ((static_cast<size_t>(b) * ltok + static_cast<size_t>(t) * p.P + row) * p.H + h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(o_tmem + 32 * c, o);
          tmem_wait_ld_regs(o);
          if (valid) {
            uint4 pk[4];
            uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
            for (int i = 0; i < 16; ++i) pw[i] = pack_bf16x2(o[2 * i] * inv_l, o[2 * i + 1] * inv_l);
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = pk[i];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One CTA waits on a barrier that nothing arrives on; the bounded wait runs out.
__global__ void watchdog_selftest_kernel(unsigned long long budget_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const Watch w{budget_ns, &abort_flag};
  (void)__all_sync(0xffffffffu, wait_bounded(&bar, 0, w));
}

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

// [batch][tokens][heads*d] bf16 viewed as a 3-D tensor {heads*d, tokens, batch};
// one box = 64 columns (128 bytes, one swizzle row) x 128 tokens.
bool make_map(CUtensorMap* tm, const void* base, int B, long long tokens, int H, int d) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(H) * d, static_cast<cuuint64_t>(tokens),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * d * 2, static_cast<cuuint64_t>(tokens) * H * d * 2};
  cuuint32_t box[3] = {64, kBM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

std::mutex g_attr_mu;
bool g_attr_set[2][64] = {};

template <int D>
lvsa_status launch(const KernelParams& kp, int B, cudaStream_t stream, int dev) {
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
  dim3 grid(static_cast<unsigned>(kp.T * kp.qtiles), static_cast<unsigned>(kp.H), static_cast<unsigned>(B));
  lvsa_attention_kernel<D><<<grid, kThreads, Cf::kSmemBytes, stream>>>(kp);
  return cudaGetLastError() == cudaSuccess ? LVSA_OK : LVSA_ERR_CUDA;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

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
  if (heads > 65535 || batch > 65535) return LVSA_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * P > INT_MAX) return LVSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return LVSA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return LVSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lists) & 3u))
    return LVSA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return LVSA_ERR_UNSUPPORTED;
  const int qtiles = (P + kBM - 1) / kBM;
  if (static_cast<long long>(T) * qtiles > INT_MAX) return LVSA_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LVSA_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return LVSA_ERR_CUDA;
  if (major != 10) return LVSA_ERR_UNSUPPORTED;

  KernelParams kp;
  const long long tokens = static_cast<long long>(T) * P;
  if (!make_map(&kp.tm_q, q, batch, tokens, heads, d) || !make_map(&kp.tm_k, k, batch, tokens, heads, d) ||
      !make_map(&kp.tm_v, v, batch, tokens, heads, d))
    return LVSA_ERR_CUDA;
  kp.out = static_cast<__nv_bfloat16*>(out);
  kp.lists = lists;
  kp.T = T;
  kp.P = P;
  kp.H = heads;
  kp.L = L;
  kp.qtiles = qtiles;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  kp.scale_log2 = sc * 1.4426950408889634f;
  kp.wait_ns = g_wait_ns;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch<128>(kp, batch, st, dev) : launch<64>(kp, batch, st, dev);
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
  lvsa::g_wait_ns = ns < 1000ull ? 1000ull : ns;
  return LVSA_OK;
}

extern "C" lvsa_status lvsa_watchdog_selftest(unsigned long long budget_ns, void* stream) {
  if (budget_ns < 1000ull) budget_ns = 1000ull;
  if (budget_ns > 10000000000ull) return LVSA_ERR_INVALID_ARG;
  lvsa::watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_ns);
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
