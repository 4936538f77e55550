// Device code of the LVSA attention path for B200 (sm_100a): the attention kernel and its helpers.
//
// "LVSA: Training-Free Sparse Attention for Long Video Diffusion" (gist.science technical summary,
// section 2 "Core Mechanism" and "Complexity"): a query token of frame t attends only to the tokens of the
// frames in A(t); one softmax over all of them; cost O(T * C * P^2 * d).
//
// One CTA per (256-row query block, head, batch entry); 384 threads.  In a joint video + text sequence
// the text query rows take blocks of their own that attend every frame, and every block's walk ends with
// one run over the text tokens (the reading taken where the pages are silent on non-video tokens).
//   warp 8      TMA producer: both 128-row Q tiles once, then K and V tiles of the frames the block
//               attends into a 5-slot shared-memory ring.  A block may hold the end of frame fa and the
//               start of fa + 1; it attends the union of their lists, walked as runs of consecutive
//               frames (one contiguous token range each, cut into 128-token tiles).  In a block of one
//               frame every row attends every run, so a tile may span the end of one run and the start of
//               the next (loaded in 8-row boxes); otherwise each run's last tile is partial.  The gather is
//               done by TMA coordinates: no mask is ever materialised.  The producer alone walks the lists
//               and publishes a record per tile (valid keys, membership, last tile) that the MMA and
//               softmax warps read.
//   warp 9      TMEM allocator and tcgen05.mma issuer (one elected lane):
//                 S_i = Q_i K_j^T  into query tile i's S columns (SS form)
//                 O_i += P_i V_j   with P_i read from TMEM (TS form), in two halves of 64 keys
//               in the order PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so the tensor core works on one
//               query tile while the other tile's softmax runs.
//   warps 0-3   softmax of query tile 0, warps 4-7 of query tile 1, one thread per row (TMEM lane):
//               online softmax in the exp2 domain with a lazily updated running max (O in TMEM is
//               rescaled only when the max grows by more than 2^8), P written back over the S columns
//               as bf16; rows of the other frame skip the tiles their frame does not attend.  On full
//               tiles the exponentials start with the running max as soon as the first 32 columns of S
//               are loaded; the max of keys 64..127 is computed alongside them, and keys 0..63 are
//               checked through their row sum (a row whose max grew by more than 2^8 has its first 64
//               keys redone), so neither the rest of the load nor the max waits in front of the
//               exponentials.
//               Epilogue O / l -> bf16 -> HBM.  The output rows may be split by token range over several
//               buffers, other GPUs' included (sequence-parallel use): each row is stored straight into
//               the buffer of the rank that owns its tokens, so the attention and the head-to-sequence
//               exchange after it are one kernel.
// Every wait is bounded: when its time budget runs out the CTA stops, sets a device status bit, lets its
// in-flight copies and MMAs finish and frees TMEM.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <cmath>

#include "lvsa.h"
#include "sm100.cuh"

__device__ unsigned int g_lvsa_dev_status = 0;

namespace lvsa {
using namespace sm100;

constexpr int kBM = 128;          // query rows per tile = MMA M
constexpr int kBN = 128;          // keys per K/V tile = largest MMA N of QK^T
constexpr int kQTiles = 2;        // query tiles per CTA, sharing every K/V tile
constexpr int kThreads = 384;     // warps 0-3: softmax tile 0, 4-7: softmax tile 1, 8: TMA, 9: MMA, 10-11 idle
// Registers: launched at 168 per thread (384 x 168 = 64512); the TMA/MMA warpgroup drops to 56 and the
// two softmax warpgroups rise to 224: 2 x 128 x 224 + 128 x 56 = 64512 (the softmax then needs no spill).
constexpr uint32_t kRegsSoftmax = 224;
constexpr uint32_t kRegsControl = 56;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kTmemCols = 512;    // S/P of tile i: columns [128 i, 128 i + 128); O of tile i: [256 + 128 i, ...)
constexpr int kOCol0 = 256;
constexpr int kChunkBytes = kBM * 128;    // one 128-byte-wide swizzle column of a 128-row tile
constexpr float kRescaleLog2 = 8.0f;      // rescale O only when the max grows by > 2^8
constexpr float kRescaleSum = 256.0f;     // 2^kRescaleLog2

constexpr int kMaxT = 4096;               // latent frames supported (frame bitmaps in shared memory)
constexpr int kMaxChunks = 64;            // output buffers a launch can route rows to (token ranges)
constexpr int kMapWords = kMaxT / 32;

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kSlots = (D == 128) ? 5 : 10;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kQTiles * kTileBytes;
  static constexpr int kOffBar = kOffRing + kSlots * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kOffMap = kOffBar + kBarBytes;             // two frame bitmaps of kMapWords words
  static constexpr int kSmemBytes = kOffMap + 2 * kMapWords * 4 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(8 * (1 + 2 * kSlots + 9) + 8 <= kBarBytes, "barrier area");
};

struct KernelParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_k8;  // K and V with 8-row boxes: tiles that span two runs are loaded in 8-row pieces
  CUtensorMap tm_v8;
  int pack;           // frames hold a multiple of 8 tokens and there is no text: single-frame blocks pack tiles
  const int32_t* lists;
  int T, P, H, L;    // H: heads in this launch (grid.y)
  int ntext;         // text tokens after the T*P video tokens (joint sequence); 0: video only
  int nvblocks;      // CTAs of video query rows per (batch, head); the text query rows take the rest
  int HS;            // heads per token row of an output buffer (H for a whole tensor, more for a band)
  int head0;         // output head of this launch's head 0 within such a row
  int nchunks;       // output rows are split by token range over nchunks buffers
  int routed;        // 1: some output buffers are another GPU's memory (stores released at system scope)
  int chunk_start[kMaxChunks + 1];           // buffer c holds tokens [chunk_start[c], chunk_start[c + 1])
  __nv_bfloat16* out_chunk[kMaxChunks];      // of every batch entry: [batch][tokens of c][HS][d]
  int straddle;      // 1: CTA c takes query rows [256c, 256c+256) of the whole frame-major sequence
  int qblocks;       // straddle == 0: ceil(P / 256) CTAs per query frame
  int nblocks;       // query blocks per (batch, head)
  int block0;        // query block of blockIdx.x == 0 (a launch may cover a range of the blocks)
  float scale_log2;  // softmax scale * log2(e)
  long long wait_cycles;
};

// ------------------------------------------------------------------ bounded waits
// The budget is counted in SM clock cycles (the host converts a ns budget at 2 GHz,
// so at lower clocks it lasts longer in wall time).  The cycle counter and the abort
// flag are only looked at every 64 polls: the poll itself must stay cheap, since
// a slow poll delays the hand-off it waits for.

struct Watch {
  long long budget_cycles;
  volatile int* abort_flag;  // shared memory, CTA-wide
};

// Returns false when the budget ran out (status bit set) or another role of the
// CTA already gave up.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const Watch& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*w.abort_flag) return false;
      if (clock64() - t0 > w.budget_cycles) {
        *w.abort_flag = 1;
        atomicOr(&g_lvsa_dev_status, LVSA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// Used only while shutting down after an abort: ignores the abort flag.  Copies and
// MMAs in flight always complete on their own, so the drain allows at least ~1 s
// whatever the caller's wait budget: a CTA must not exit while a copy can still land
// in its shared memory.
constexpr long long kMinDrainCycles = 2000000000ll;

__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, long long budget_cycles) {
  budget_cycles = budget_cycles > kMinDrainCycles ? budget_cycles : kMinDrainCycles;
  const long long t0 = clock64();
  for (uint32_t it = 0; !mbar_try_wait(bar, parity); ++it) {
    if ((it & 63u) == 63u && clock64() - t0 > budget_cycles) {
      atomicOr(&g_lvsa_dev_status, LVSA_DEV_TIMEOUT);
      return;
    }
  }
}

// ------------------------------------------------------------------ K/V tile walk
// The CTA's query rows belong to frame fa, or to frames fa and fb = fa + 1.  Their
// frame lists are held as bitmaps over [0, T) (so list order and duplicates do not
// matter).  The walk visits the union in ascending frame order as runs of
// consecutive frames with the same membership (bit 0: attended by fa, bit 1: by
// fb); a run is one contiguous token range, cut into tiles of at most 128 tokens
// (in a packed walk a tile may take the end of one run and the start of the next).
// Only the TMA producer walks; the other roles read the tile records it publishes.
struct FrameWalk {
  const uint32_t* ma;
  const uint32_t* mb;
  int T, P, nwords, ntext;
  int f = 0, pos = 0, end = 0, mask = 0;
  bool text_done = false;

  __device__ FrameWalk(const uint32_t* a, const uint32_t* b_, int T_, int P_, int ntext_)
      : ma(a), mb(b_), T(T_), P(P_), nwords((T_ + 31) >> 5), ntext(ntext_) {}

  // After the frames: the text tokens of a joint sequence, one run that every query row attends.
  __device__ __forceinline__ bool text_run() {
    if (text_done || ntext <= 0) return false;
    text_done = true;
    pos = T * P;
    end = T * P + ntext;
    mask = 3;
    return true;
  }

  __device__ __forceinline__ int bits(int g) const {
    return static_cast<int>(((ma[g >> 5] >> (g & 31)) & 1u) | (((mb[g >> 5] >> (g & 31)) & 1u) << 1));
  }

  // tiles of a packed walk may span two runs; the last tile's second run starts at token tok_b after n_a
  // tokens of the first (n_a == the tile's tokens when it lies in one run)
  bool pack = false;
  int tok_b = 0, n_a = 0;

  __device__ __forceinline__ bool next(int& tok, int& nvalid, int& tmask) {
    if (!next_run()) return false;
    tok = pos;
    nvalid = min(kBN, end - pos);
    tmask = mask;
    pos += nvalid;
    n_a = nvalid;
    if (pack && nvalid < kBN && next_run()) {
      tok_b = pos;
      const int nb = min(kBN - nvalid, end - pos);
      pos += nb;
      nvalid += nb;
      tmask &= mask;
    }
    return true;
  }

  // makes [pos, end) the rest of the current run or the next non-empty run; false after the last
  __device__ __forceinline__ bool next_run() {
    while (pos >= end) {
      if (f >= T) {
        if (text_run()) continue;
        return false;
      }
      int wi = f >> 5;
      uint32_t word = (ma[wi] | mb[wi]) & (0xffffffffu << (f & 31));
      bool none = false;
      while (word == 0) {
        if (++wi >= nwords) {
          none = true;
          break;
        }
        word = ma[wi] | mb[wi];
      }
      const int f0 = none ? T : (wi << 5) + __ffs(word) - 1;
      if (f0 >= T) {
        f = T;
        if (text_run()) continue;
        return false;
      }
      const int m0 = bits(f0);
      int f1 = f0;
      while (f1 + 1 < T && bits(f1 + 1) == m0) ++f1;
      pos = f0 * P;
      end = (f1 + 1) * P;
      mask = m0;
      f = f1 + 1;
    }
    return true;
  }
};

// ------------------------------------------------------------------ tile records
// The producer walks the frame lists once and publishes, for K/V tile j, a record at entry j % kMetaSlots:
// bits 16..31 j mod 2^16, bit 10 "last tile", bits 2..9 valid keys nv (0: the walk holds no tile at all),
// bits 0..1 the membership mask of the tile's frames.  The producer is at most a few tiles ahead of any
// reader (the K/V ring bounds it), so 16 entries are never overwritten before they are read.
constexpr int kMetaSlots = 16;
__device__ __forceinline__ uint32_t tile_record(int j, int nv, int tmask, bool last) {
  return (static_cast<uint32_t>(j & 0xffff) << 16) | (last ? 1024u : 0u) | (static_cast<uint32_t>(nv) << 2) |
         static_cast<uint32_t>(tmask);
}
__device__ __forceinline__ int rec_nv(uint32_t r) { return static_cast<int>((r >> 2) & 0xff); }
__device__ __forceinline__ int rec_mask(uint32_t r) { return static_cast<int>(r & 3); }
__device__ __forceinline__ bool rec_last(uint32_t r) { return (r & 1024u) != 0; }

// Waits (bounded) until tile j's record is published; false when the budget ran out or the CTA gave up.
__device__ __forceinline__ bool read_record(volatile uint32_t* meta, int j, const Watch& w, uint32_t& rec) {
  rec = meta[j % kMetaSlots];
  if ((rec >> 16) == static_cast<uint32_t>(j & 0xffff)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    rec = meta[j % kMetaSlots];
    if ((rec >> 16) == static_cast<uint32_t>(j & 0xffff)) return true;
    if ((it & 63u) == 0) {
      if (*w.abort_flag) return false;
      if (clock64() - t0 > w.budget_cycles) {
        *w.abort_flag = 1;
        atomicOr(&g_lvsa_dev_status, LVSA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ softmax of one S tile
// Exponentials of chunk c (32 keys) of the row: P as bf16 pairs over the S columns, row sum into acc.
__device__ __forceinline__ void exp_store_chunk(uint32_t s_tmem, const float* sc, float2 scale2, float2 negm2,
                                                float2* acc, int c) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 x = ffma2(make_float2(sc[2 * i], sc[2 * i + 1]), scale2, negm2);
    float2 e;
    e.x = ex2(x.x);
    e.y = ex2(x.y);
    acc[i & 3] = fadd2(acc[i & 3], e);
    pk[i] = pack_bf16x2(e.x, e.y);
  }
  tmem_st16(s_tmem + 16 * c, pk);
}

__device__ __forceinline__ float row_max64(const float* s) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = s[k];
#pragma unroll
  for (int i = 8; i < 56; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[i + k], s[i + 8 + k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], s[56 + k]);
  return fmaxf(fmax3(a[0], a[1], a[2]), fmax3(fmax3(a[3], a[4], a[5]), a[6], a[7]));
}

__device__ __forceinline__ float row_max128(const float* s) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = s[k];
#pragma unroll
  for (int i = 8; i < 120; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[i + k], s[i + 8 + k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], s[120 + k]);
  return fmaxf(fmax3(a[0], a[1], a[2]), fmax3(fmax3(a[3], a[4], a[5]), a[6], a[7]));
}

// Thread = one query row.  Loads the row of S from TMEM, masks columns past the
// run end, updates the running max lazily (rescaling the row of O in TMEM when
// needed), writes P = 2^(scale*log2e*s - m) as bf16 over the S columns and
// returns the row sum of P through `l`.  `skip`: the row's frame does not attend
// the tile (P = 0, max and sum unchanged).  After the first 64 keys of P are
// stored it arrives on `bar_half`, so the tensor core can run the first half of
// PV while this thread computes the second half.
template <int D>
__device__ __forceinline__ bool softmax_tile(uint32_t s_tmem, uint32_t o_tmem, int nv, int j, bool skip, float sl2,
                                             float& m, float& l, uint64_t* bar_o, const Watch& w, uint64_t* bar_half) {
  float s[kBN];
  // Speculative path (full tiles, every row of the warp with a finite running max or skipping the tile):
  // the exponentials start with the running max as soon as keys 0..31 are loaded, and the tile max is
  // computed alongside; a warp with a row whose max grew by more than 2^8 redoes keys 0..63 with the new
  // max before handing them over.
  if (nv == kBN && __all_sync(0xffffffffu, m != -INFINITY || skip)) {
    const float2 scale2 = make_float2(sl2, sl2);
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    tmem_ld32(s_tmem + 0, s + 0);
    tmem_wait_ld_regs(s + 0);
    tmem_ld32(s_tmem + 32, s + 32);
    tmem_ld32(s_tmem + 64, s + 64);
    tmem_ld32(s_tmem + 96, s + 96);
    float2 negm2 = skip ? make_float2(-INFINITY, -INFINITY) : make_float2(-m, -m);
    exp_store_chunk(s_tmem, s + 0, scale2, negm2, acc, 0);
    tmem_wait_ld_regs(s + 32);
    tmem_wait_ld_regs(s + 64);
    tmem_wait_ld_regs(s + 96);
    // keys 64..127: their max; keys 0..63: a key more than 2^8 above the running max makes its P, and so
    // the row sum of keys 0..63, exceed 2^8 -- only then is their max needed
    const float hi_max = skip ? -INFINITY : row_max64(s + 64) * sl2;
    exp_store_chunk(s_tmem, s + 32, scale2, negm2, acc, 1);
    const float2 lo01 = fadd2(acc[0], acc[1]);
    const float2 lo23 = fadd2(acc[2], acc[3]);
    const float2 lo = fadd2(lo01, lo23);
    const bool check = hi_max > m + kRescaleLog2 || lo.x + lo.y > kRescaleSum;
    if (__any_sync(0xffffffffu, check)) {
      const float tile_max = skip ? -INFINITY : fmaxf(row_max64(s) * sl2, hi_max);
      float alpha = 1.f;
      if (tile_max > m + kRescaleLog2) {
        alpha = ex2(m - tile_max);
        l *= alpha;
        m = tile_max;
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!__all_sync(0xffffffffu, wait_bounded(bar_o, (j - 1) & 1, w))) return false;
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
      // keys 0..63 again with the new max (after the first stores of those columns have completed)
      tmem_wait_st();
      negm2 = skip ? make_float2(-INFINITY, -INFINITY) : make_float2(-m, -m);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
      exp_store_chunk(s_tmem, s + 0, scale2, negm2, acc, 0);
      exp_store_chunk(s_tmem, s + 32, scale2, negm2, acc, 1);
    }
    // keys 0..63 of P are in TMEM: the MMA warp may start the first half of PV
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bar_half);
    exp_store_chunk(s_tmem, s + 64, scale2, negm2, acc, 2);
    exp_store_chunk(s_tmem, s + 96, scale2, negm2, acc, 3);
    const float2 t01 = fadd2(acc[0], acc[1]);
    const float2 t23 = fadd2(acc[2], acc[3]);
    const float2 tt = fadd2(t01, t23);
    l += tt.x + tt.y;
    return true;
  }
  tmem_ld32(s_tmem + 0, s + 0);
  if (nv > 32) tmem_ld32(s_tmem + 32, s + 32);
  if (nv > 64) tmem_ld32(s_tmem + 64, s + 64);
  if (nv > 96) tmem_ld32(s_tmem + 96, s + 96);
  tmem_wait_ld_regs(s + 0);
  tmem_wait_ld_regs(s + 32);
  tmem_wait_ld_regs(s + 64);
  tmem_wait_ld_regs(s + 96);
  const bool partial = nv < kBN;
  if (partial) {
#pragma unroll
    for (int i = 0; i < kBN; ++i)
      if (i >= nv) s[i] = -INFINITY;
  }
  // row max: 8 chains of 3-input max
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = s[k];
#pragma unroll
  for (int i = 8; i < 120; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[i + k], s[i + 8 + k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], s[120 + k]);
  // a row whose frame does not attend this tile's frames takes no part in it:
  // its max stays and its P is 2^-inf = 0
  const float tile_max =
      skip ? -INFINITY : fmaxf(fmax3(a[0], a[1], a[2]), fmax3(fmax3(a[3], a[4], a[5]), a[6], a[7])) * sl2;

  float alpha = 1.f;
  if (tile_max > m + kRescaleLog2) {
    alpha = ex2(m - tile_max);
    l *= alpha;
    m = tile_max;
  }
  if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
    // O holds PV(0..j-1): wait for PV(j-1), then rescale this thread's row
    if (!__all_sync(0xffffffffu, wait_bounded(bar_o, (j - 1) & 1, w))) return false;
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

  const float2 scale2 = make_float2(sl2, sl2);
  const float2 negm2 = skip ? make_float2(-INFINITY, -INFINITY) : make_float2(-m, -m);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (c == 0 || nv > 32 * c) {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 x = ffma2(make_float2(s[32 * c + 2 * i], s[32 * c + 2 * i + 1]), scale2, negm2);
        float2 e;
        e.x = ex2(x.x);
        e.y = ex2(x.y);
        acc[i & 3] = fadd2(acc[i & 3], e);
        pk[i] = pack_bf16x2(e.x, e.y);
      }
      tmem_st16(s_tmem + 16 * c, pk);  // P overwrites the first half of the S columns
    }
    if (c == 1) {
      // keys 0..63 of P are in TMEM: the MMA warp may start the first half of PV
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_half);
    }
  }
  const float2 t01 = fadd2(acc[0], acc[1]);
  const float2 t23 = fadd2(acc[2], acc[3]);
  const float2 tt = fadd2(t01, t23);
  l += tt.x + tt.y;
  return true;
}

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
  uint64_t* bar_s = bar_empty + Cf::kSlots;  // [2] S_i(j) ready in TMEM
  uint64_t* bar_p = bar_s + 2;               // [2] P_i(j) written to TMEM (128 arrivals)
  uint64_t* bar_o = bar_p + 2;               // [2] PV_i(j) finished
  uint64_t* bar_ph = bar_o + 2;              // [2] P_i(j) keys 0..63 written (128 arrivals)
  uint64_t* bar_drain = bar_ph + 2;          // all MMAs of the CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  // K/V tile records written by the producer (tile j at entry j % kMetaSlots; see tile_record)
  volatile uint32_t* tile_meta = reinterpret_cast<volatile uint32_t*>(bars + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int vtok = p.T * p.P;      // video tokens
  const int ltok = vtok + p.ntext;  // all tokens of a sequence
  // query rows [r0, r1): video rows of one frame fa, or of fa and fb = fa + 1; or text rows (text_rows),
  // which attend every frame
  int r0, r1;
  const int qblk = blockIdx.x + p.block0;  // this CTA's query block
  const bool text_rows = qblk >= p.nvblocks;
  if (text_rows) {
    r0 = vtok + (qblk - p.nvblocks) * (kQTiles * kBM);
    r1 = min(r0 + kQTiles * kBM, ltok);
  } else if (p.straddle) {
    r0 = qblk * (kQTiles * kBM);
    r1 = min(r0 + kQTiles * kBM, vtok);
  } else {
    const int qb = qblk % p.qblocks;
    const int t = qblk / p.qblocks;
    r0 = t * p.P + qb * (kQTiles * kBM);
    r1 = min(r0 + kQTiles * kBM, (t + 1) * p.P);
  }
  const int fa = text_rows ? p.T : r0 / p.P;
  const int fb = text_rows ? p.T : (r1 - 1) / p.P;
  const bool has1 = r0 + kBM < r1;  // the second query tile has rows
  const bool pack = p.pack && fa == fb && !text_rows;  // every row of the block attends every run
  uint32_t* map_a = reinterpret_cast<uint32_t*>(smem + Cf::kOffMap);
  uint32_t* map_b = map_a + kMapWords;
  {
    // frame bitmaps of the lists of fa and fb (map_b stays empty when fb == fa)
    const int nwords = (p.T + 31) >> 5;
    for (int i = threadIdx.x; i < nwords; i += kThreads) {
      // text rows: every frame [0, T) in both maps (every run attended by every row)
      const uint32_t all = (i < (p.T >> 5)) ? 0xffffffffu : ((1u << (p.T & 31)) - 1u);
      map_a[i] = text_rows ? all : 0u;
      map_b[i] = text_rows ? all : 0u;
    }
    __syncthreads();
    bool bad = false;
    const int32_t* la = p.lists + static_cast<size_t>(fa) * p.L;
    const int32_t* lb = p.lists + static_cast<size_t>(fb) * p.L;
    const int nset = text_rows ? 0 : (fb != fa) ? 2 * p.L : p.L;
    for (int i = threadIdx.x; i < nset; i += kThreads) {
      const int f = (i < p.L) ? __ldg(la + i) : __ldg(lb + (i - p.L));
      if (f < 0 || f >= p.T) {
        bad = true;
        continue;
      }
      atomicOr((i < p.L ? map_a : map_b) + (f >> 5), 1u << (f & 31));
    }
    if (bad) atomicOr(&g_lvsa_dev_status, LVSA_DEV_BAD_LIST);
  }

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < Cf::kSlots; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s + i, 1);
      mbar_init(bar_p + i, 4 * 32);
      mbar_init(bar_o + i, 1);
      mbar_init(bar_ph + i, 4 * 32);
    }
    mbar_init(bar_drain, 1);
    for (int i = 0; i < kMetaSlots; ++i) tile_meta[i] = 0xffff0000u;
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
  const Watch w{p.wait_cycles, abort_flag};

  if (warp >= 8) {
  regs_dec<kRegsControl>();
  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the list (warp-uniform control flow); one elected
    // lane arms the barriers and issues the copies.
    const int col0 = h * D;
    const int qrow = r0;
    if (elect_one()) {
      mbar_arrive_expect_tx(bar_q, (has1 ? 2 : 1) * Cf::kTileBytes);
#pragma unroll
      for (int c = 0; c < Cf::kChunks; ++c) tma_load_3d(sQ + c * kChunkBytes, &p.tm_q, bar_q, col0 + c * 64, qrow, b);
      if (has1) {
#pragma unroll
        for (int c = 0; c < Cf::kChunks; ++c)
          tma_load_3d(sQ + Cf::kTileBytes + c * kChunkBytes, &p.tm_q, bar_q, col0 + c * 64, qrow + kBM, b);
      }
    }
    __syncwarp();
    int issued = 0;
    int slot = 0;         // ring slot and phase of the next load
    uint32_t phase = 0;
    bool ok = true;
    auto load = [&](const CUtensorMap* tm, const CUtensorMap* tm8, int tok, int n_a, int tok_b) {
      if (!__all_sync(0xffffffffu, wait_bounded(bar_empty + slot, phase ^ 1, w))) {
        ok = false;
        return;
      }
      if (elect_one()) {
        mbar_arrive_expect_tx(bar_full + slot, Cf::kTileBytes);
        uint8_t* dst = sRing + slot * Cf::kTileBytes;
        if (tok_b == 0) {
#pragma unroll
          for (int c = 0; c < Cf::kChunks; ++c)
            tma_load_3d(dst + c * kChunkBytes, tm, bar_full + slot, col0 + c * 64, tok, b);
        } else {
          // a tile across two runs: rows [0, n_a) from tok, rows [n_a, 128) from tok_b, in 8-row boxes
          // (1024 bytes of a 64-column chunk each, so every box lands on a swizzle-atom boundary)
          // (the box loop stays rolled: unrolled, its 32 coordinates spill the 56 registers of this warp)
          const int ga = n_a >> 3;
#pragma unroll 1
          for (int g = 0; g < kBN / 8; ++g) {
            const int row = g < ga ? tok + 8 * g : tok_b + 8 * (g - ga);
#pragma unroll
            for (int c = 0; c < Cf::kChunks; ++c)
              tma_load_3d(dst + c * kChunkBytes + g * 1024, tm8, bar_full + slot, col0 + c * 64, row, b);
          }
        }
      }
      __syncwarp();
      ++issued;
      if (++slot == Cf::kSlots) {
        slot = 0;
        phase ^= 1;
      }
    };
    // consumption order of the MMA warp: K0, V0, K1, V1, ...
    FrameWalk walk(map_a, map_b, p.T, p.P, p.ntext);
    walk.pack = pack;
    int tok, nv, tmask;
    bool have = walk.next(tok, nv, tmask);
    int n_a = walk.n_a, tok_b = walk.n_a < nv ? walk.tok_b : 0;
    if (!have && lane == 0) tile_meta[0] = tile_record(0, 0, 0, true);  // no tile at all
    for (int j = 0; ok && have; ++j) {
      int tok_n, nv_n, tmask_n;
      const bool more = walk.next(tok_n, nv_n, tmask_n);
      const int n_a_n = walk.n_a, tok_b_n = walk.n_a < nv_n ? walk.tok_b : 0;
      if (lane == 0) tile_meta[j % kMetaSlots] = tile_record(j, nv, tmask, !more);
      __syncwarp();  // the record is written before the loads' barrier arrivals
      load(&p.tm_k, &p.tm_k8, tok, n_a, tok_b);
      if (ok) load(&p.tm_v, &p.tm_v8, tok, n_a, tok_b);
      n_a = n_a_n;
      tok_b = tok_b_n;
      tok = tok_n;
      nv = nv_n;
      tmask = tmask_n;
      have = more;
    }
    if (!ok) {
      // stopped early: let every copy still in flight land before the CTA exits
      wait_drain(bar_q, 0, p.wait_cycles);
      const int first = issued > Cf::kSlots ? issued - Cf::kSlots : 0;
      for (int i = first; i < issued; ++i) wait_drain(bar_full + i % Cf::kSlots, (i / Cf::kSlots) & 1, p.wait_cycles);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Per K/V tile j:  PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1): while softmax 1 works on S_1(j)
    // the tensor core runs tile 0's products, and the other way round.  Each PV is issued in two
    // halves (keys 0..63 as soon as the softmax has stored them, then keys 64..127).  The whole warp
    // runs the schedule (descriptors stay warp-uniform); one elected lane issues each group of MMAs and
    // the commits that follow it.  The issuer shares a sub-partition with a softmax warp of each
    // warpgroup, so its instruction count sits on the P hand-off chain: descriptors are built as 32-bit
    // low words, there is one elected block per group rather than per MMA, and the tile sequence comes
    // from the producer's records instead of a walk of the lists.
    const uint32_t sq = smem_u32(sQ);
    const uint32_t sr = smem_u32(sRing);
    const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
    // descriptor of a K-major Q/K tile at byte address a; + (kk>>2)*16 KB + (kk&3)*32 B per 16-wide k-step
    const uint64_t kdesc0 = smem_desc_sw128(0, 16, 1024);
    // descriptor of an MN-major V tile: 64-wide d chunks 16 KB apart (LBO), 8-key groups 1 KB apart (SBO)
    const uint64_t vdesc0 = smem_desc_sw128(0, kChunkBytes, 1024);
    const uint32_t khi = static_cast<uint32_t>(kdesc0 >> 32), klo0 = static_cast<uint32_t>(kdesc0);
    const uint32_t vhi = static_cast<uint32_t>(vdesc0 >> 32), vlo0 = static_cast<uint32_t>(vdesc0);
    auto qk = [&](int i, uint32_t k_addr, int n_mma) {
      const uint32_t qd = klo0 + ((sq + i * Cf::kTileBytes) >> 4);
      const uint32_t kd = klo0 + (k_addr >> 4);
      const uint32_t idesc = idesc_bf16_f32(kBM, n_mma, false);
      mma_qk_group<D>(tmem + 128 * i, qd, kd, khi, idesc, 0u);
    };
    auto pv = [&](int i, uint32_t v_addr, int n_mma, bool accumulate, int k_lo, int k_hi) {
      const uint32_t vd = vlo0 + (v_addr >> 4);
      if (n_mma >= 16 * k_hi) {  // the four 16-key steps of this half are all in the tile
        mma_pv_group4(tmem + kOCol0 + 128 * i, tmem + 128 * i + k_lo * 8, vd + ((k_lo * 16 * 128) >> 4), vhi,
                      idesc_pv, (accumulate || k_lo > 0) ? 1u : 0u);
        return;
      }
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk) {
        if (kk < k_lo) continue;
        if (kk >= k_hi || kk * 16 >= n_mma) break;
        mma_ts_lo(tmem + kOCol0 + 128 * i, tmem + 128 * i + kk * 8, vd + ((kk * 16 * 128) >> 4), vhi, idesc_pv,
                  (accumulate || kk > 0) ? 1u : 0u);
      }
    };
    auto commit = [&](uint64_t* bar) { mma_commit(bar); };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_bounded(bar, parity, w));
    };
    // ring slot and phase of the next load consumed, advanced by one per load (consumption order K0, V0, K1, ...)
    int rslot = 0;
    uint32_t rphase = 0;
    auto take = [&](int& slot, uint32_t& phase) {
      slot = rslot;
      phase = rphase;
      if (++rslot == Cf::kSlots) {
        rslot = 0;
        rphase ^= 1;
      }
    };
    bool ok = wait_all(bar_q, 0);
    uint32_t rec = 0;
    if (ok) ok = __all_sync(0xffffffffu, read_record(tile_meta, 0, w, rec));
    if (ok && rec_nv(rec) > 0) {
      int n_cur = (rec_nv(rec) + 15) & ~15;
      int k0;
      uint32_t k0p;
      take(k0, k0p);
      ok = wait_all(bar_full + k0, k0p);
      if (ok) {
        tc_fence_after();
        const uint32_t k_addr = sr + k0 * Cf::kTileBytes;
        if (elect_one()) {
          qk(0, k_addr, n_cur);
          commit(bar_s + 0);
          if (has1) {
            qk(1, k_addr, n_cur);
            commit(bar_s + 1);
          }
          commit(bar_empty + k0);
        }
        __syncwarp();
      }
      for (int j = 0; ok; ++j) {
        const bool has_next = !rec_last(rec);
        int n_next = 0;
        int vi;
        uint32_t vph;
        take(vi, vph);
        const uint32_t v_addr = sr + vi * Cf::kTileBytes;
        if (!wait_all(bar_ph + 0, j & 1) || !wait_all(bar_full + vi, vph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) pv(0, v_addr, n_cur, j > 0, 0, 4);
        __syncwarp();
        // the next K tile is waited for while the softmax finishes P_0(j), so that nothing but the
        // P_0 hand-off stands between PV_0(j) and QK_0(j+1); commits that nobody waits on soon go
        // after the next group of MMAs
        int ki = -1;
        uint32_t k_addr = 0;
        if (has_next) {
          uint32_t kph;
          take(ki, kph);
          k_addr = sr + ki * Cf::kTileBytes;
          if (!wait_all(bar_full + ki, kph)) {
            ok = false;
            break;
          }
          // the next tile's record was written before its K load was armed
          rec = tile_meta[(j + 1) % kMetaSlots];
          n_next = (rec_nv(rec) + 15) & ~15;
        }
        if (!wait_all(bar_p + 0, j & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          pv(0, v_addr, n_cur, j > 0, 4, 8);
          if (has_next) {
            qk(0, k_addr, n_next);
            commit(bar_s + 0);
          }
          commit(bar_o + 0);
          if (!has1) {
            commit(bar_empty + vi);
            if (has_next) commit(bar_empty + ki);
          }
        }
        __syncwarp();
        if (has1) {
          if (!wait_all(bar_ph + 1, j & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) pv(1, v_addr, n_cur, j > 0, 0, 4);
          __syncwarp();
          if (!wait_all(bar_p + 1, j & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            pv(1, v_addr, n_cur, j > 0, 4, 8);
            if (has_next) {
              qk(1, k_addr, n_next);
              commit(bar_s + 1);
            }
            commit(bar_o + 1);
            commit(bar_empty + vi);
            if (has_next) commit(bar_empty + ki);
          }
          __syncwarp();
        }
        if (!has_next) break;
        n_cur = n_next;
      }
    }
    // every MMA issued must be complete before TMEM is released
    if (elect_one()) commit(bar_drain);
    __syncwarp();
    wait_drain(bar_drain, 0, p.wait_cycles);
    __syncwarp();
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax + epilogue (warps 0-7)
    const int qi = warp >> 2;            // query tile of this warpgroup
    const int r = threadIdx.x & 127;     // row within the tile = TMEM lane
    if (qi == 0 || has1) {
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t s_tmem = tmem + lane_off + 128 * qi;
      const uint32_t o_tmem = tmem + lane_off + kOCol0 + 128 * qi;
      float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale by < 8)
      float l = 0.f;        // running sum of 2^(scaled s - m)
      bool ok = true;
      int j = 0;
      const int row = r0 + qi * kBM + r;  // query row in the frame-major sequence
      const int rbit = (row / p.P == fa) ? 1 : 2;
      for (;;) {
        uint32_t rec;
        ok = __all_sync(0xffffffffu, read_record(tile_meta, j, w, rec));
        if (!ok) break;
        const int nv = rec_nv(rec), tmask = rec_mask(rec);
        if (nv == 0) break;  // no tile at all
        ok = __all_sync(0xffffffffu, wait_bounded(bar_s + qi, j & 1, w));
        if (!ok) break;
        tc_fence_after();
        ok = softmax_tile<D>(s_tmem, o_tmem, nv, j, (tmask & rbit) == 0, p.scale_log2, m, l, bar_o + qi, w,
                             bar_ph + qi);
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p + qi);
        ++j;
        if (rec_last(rec)) break;
      }
      // j == 0: the block walked no tile at all (its frames have no valid list entry); O in TMEM was never
      // written, and the rows get zeros
      if (ok && j > 0) ok = __all_sync(0xffffffffu, wait_bounded(bar_o + qi, (j - 1) & 1, w));
      if (ok) {
        if (j > 0) tc_fence_after();
        const float inv_l = l > 0.f ? 1.f / l : 0.f;  // a frame with no valid list entry: zero output
        const bool valid = row < r1;
        // the buffer that holds this row's token: the last chunk starting at or before it (an empty
        // chunk is never that one, since the next chunk starts at the same token)
        int c = 0;
        for (int hi = p.nchunks - 1; c < hi;) {
          const int mid = (c + hi + 1) >> 1;
          if (p.chunk_start[mid] <= row) c = mid; else hi = mid - 1;
        }
        const int c0 = p.chunk_start[c];
        const size_t clen = static_cast<size_t>(p.chunk_start[c + 1] - c0);
        __nv_bfloat16* dst = p.out_chunk[c] + ((b * clen + (row - c0)) * p.HS + p.head0 + h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          if (j > 0) {
            tmem_ld32(o_tmem + 32 * c, o);
            tmem_wait_ld_regs(o);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          }
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
        // stores into another GPU's memory: ordered before anything the host does after this kernel
        if (p.routed) __threadfence_system();
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
__global__ void watchdog_selftest_kernel(long long budget_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const Watch w{budget_cycles, &abort_flag};
  (void)__all_sync(0xffffffffu, wait_bounded(&bar, 0, w));
}

}  // namespace lvsa
