// Fused attention forward (prefill) for sm_100a.
//
// O = softmax(scale * Q K^T + M) V and LSE per row, with M the causal mask
// when requested ("Fast Attention Kernels and Operator Fusion", section
// "FlashAttention-Style Kernels": the score block of each tile is computed,
// the softmax statistics are updated and the output is accumulated on chip,
// so the N x N score matrix never reaches HBM).  The online-softmax running
// max / running sum and the one-multiply rescale are the incremental form the
// anylearn.cc lesson describes ("Five things", second point).
//
// Persistent kernel, one 512-thread CTA per SM.  A work item is 256 query
// rows of one (batch, head): two 128-row tiles Q0 and Q1 that share every K/V
// tile brought in.  Items are ordered heaviest first (causal) and dealt to
// the CTAs in a snake order (c, then G-1-c, ...) to even out the causal work.
//   warps 0-3   softmax of Q0 (thread t owns row t = TMEM lane t)
//   warps 4-7   softmax of Q1
//   warps 8-11  epilogue: O / l -> bf16 rows and LSE, while the next item runs
//   warp 12     TMA producer: Q0/Q1 per item, K_j and V_j into 2-stage rings
//   warp 13     allocates tensor memory; lane 0 issues every tcgen05.mma
// Tensor memory (512 columns): S0 | S1 (128 fp32 columns each) | O0 | O1 (D
// columns each).  P_t (bf16 pairs) overwrites the first 64 columns of S_t and
// is the A operand of O_t += P_t V_j.  The two softmax warpgroups ping-pong:
// while one computes exponentials the tensor core runs the other tile's MMAs.
// The O rescale is lazy: the running max used for P only moves when a tile
// max exceeds it by more than 2^8, and the final O / l uses that same max,
// so the result is exact.  When S_t of tile j is complete, O_t += P_t V_{j-1}
// (issued before it) is complete too, so the softmax warps rescale O_t in
// place without a further wait.
#pragma once

#include "exp2_poly.cuh"
#include "ptx.cuh"
#include "tmem_ldst.cuh"

namespace attn {

// One column pair in every kExp2EmuPeriod takes its exp2 from a polynomial on
// the FMA pipes instead of the MUFU unit, which is otherwise as busy as the
// tensor core (0 disables it).
#ifndef ATTN_EXP2_EMU_PERIOD
#define ATTN_EXP2_EMU_PERIOD 0
#endif
constexpr int kExp2EmuPeriod = ATTN_EXP2_EMU_PERIOD;
// The FP8 kernels halve the tensor-core time per tile, so the exponentials
// weigh more: there one group of four in eight takes the polynomial
// (measured +2 % on the causal workloads; the bf16 kernels lose with it).
#ifndef ATTN_EXP2_EMU_PERIOD_FP8
#define ATTN_EXP2_EMU_PERIOD_FP8 8
#endif
constexpr int kExp2EmuPeriodFp8 = ATTN_EXP2_EMU_PERIOD_FP8;



// 2^x by range reduction x = n + f, n = round(x), |f| <= 1/2: adding
// 1.5*2^23 rounds x to an integer held in the low mantissa bits, 2^f comes
// from the fitted cubic (exp2_poly.cuh) and n is added to the exponent field.
// x is clamped at -126 so the exponent never underflows past zero.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  float q = fmaf(kExp2C3, f, kExp2C2);
  q = fmaf(q, f, kExp2C1);
  q = fmaf(q, f, kExp2C0);
  // (bits(t) - bits(1.5*2^23)) << 23 == bits(t) << 23: the constant's low 9 bits are 0.
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

struct PrefillParams {
  __nv_bfloat16* o;  // [B, Hq, N, D]; paged: [total_q, Hq, D]
  float* lse;        // [B, Hq, N];    paged: [total_q, Hq]
  int B, Hq, Hkv, N;
  int group;         // Hq / Hkv
  int num_m;         // ceil(N / 256): 256-row query blocks per head
  int num_items;     // B * Hq * num_m (paged: counted on the device)
  int window_left;   // query i sees keys >= i - window_left (kernels with WINDOW only)
  float scale_log2;  // scale * log2(e) (FP8: times the Q and K descales)
  float scale;       // the softmax scale itself (additive M only)
  float o_scale;     // FP8: the V descale, applied to O in the epilogue
  // Paged prefill (kernels with PAGED only): the new queries of sequence s
  // are packed rows cu_q[s] .. cu_q[s+1]-1; the cache holds seq_lens[s]
  // tokens of it (the new ones last), read through block_table.
  const int32_t* cu_q;         // [num_seqs + 1]
  const int32_t* seq_lens;     // [num_seqs]
  const int32_t* block_table;  // [num_seqs, max_pages]
  const __nv_bfloat16* k_pool; // [num_pages, page_size, Hkv, D] (plain loads of partial pages)
  const __nv_bfloat16* v_pool;
  int num_seqs, total_q, max_pages, num_pages, page_size;
  int page_box;                // rows per K/V TMA box: min(page_size, 128)
  // Block-sparse (kernels with SPARSE only): bit j % 64 of word j / 64 of row
  // qb of head (b, h) keeps KV tile j for query tile qb; rows of mask_words
  // words at block_mask + b * mask_b_stride + h * mask_h_stride + qb * mask_words.
  const uint64_t* block_mask;
  long long mask_b_stride, mask_h_stride;
  int mask_words;              // ceil(ceil(N / 128) / 64), at most kMaskWords
  // Additive M (kernels with BIAS only): bf16, natural-log units, row i of
  // head (b, h) at bias + b * bias_b_stride + h * bias_h_stride + i * bias_row_stride
  // (elements; rows padded to a multiple of 8, 16-byte aligned).
  const __nv_bfloat16* bias;
  long long bias_b_stride, bias_h_stride, bias_row_stride;
};

constexpr int kMaskWords = 4;  // block-sparse masks cover N <= 4 * 64 * 128 = 32768

constexpr int kPagedMaxSeqs = 1024;    // sequences per paged-prefill call
constexpr int kPagedMaxBlocks = 2048;  // 256-row query blocks per paged-prefill call

constexpr int kPrefillThreads = 512;
constexpr float kRescaleThreshold = 8.0f;  // in log2 units
// FP8: P is stored as e4m3 scaled by 2^8 (so that the weights of keys a few
// units below the row max stay normal numbers), and the stale max may lag the
// true one by at most 0.5, so 2^8 * 2^0.5 = 362 stays below e4m3's 448.
constexpr float kFp8PLog2 = 8.0f;
constexpr float kRescaleThresholdFp8 = 0.5f;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, bool PAGED = false, bool FP8 = false, bool SPARSE = false>
struct PrefillLayout {
  static_assert(!FP8 || D == 128, "FP8 tiles are one 128-byte box wide");
  static constexpr int NS = 2;                     // K and V ring depth
  static constexpr int kElemBytes = FP8 ? 1 : 2;   // bf16 or e4m3
  static constexpr int kBoxCols = 128 / kElemBytes;  // elements per 128-byte swizzled row
  static constexpr int kBoxes = D / kBoxCols;        // boxes across the head dim
  static constexpr int kBoxBytes = 128 * 128;      // 128 rows x 128 bytes (one 128B-swizzled box)
  static constexpr int kTileBytes = 128 * D * kElemBytes;
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTileBytes;
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + NS * kTileBytes;
  static constexpr int kStats = kV + NS * kTileBytes;  // float [tile 2][slot 2][m,l][128 rows]
  static constexpr int kStatsBytes = 2 * 2 * 2 * 128 * 4;
  // Paged: cached at kernel start: the query blocks in processing order
  // [kPagedMaxBlocks], cu_q [S+1], seq_lens [S], the block count and 16 ints
  // of scan scratch.
  // Block-sparse: the current item's KV-tile sets, as words in shared memory
  // (read back on use, so the loops hold none in registers): the producer's
  // union and one query tile's set per softmax warp; then two tile lists
  // (16-bit entries, up to 256 each) and their lengths, written by the lister
  // warp one item ahead of the MMA thread.
  static constexpr int kSeq = kStats + kStatsBytes;
  static constexpr int kMaskProd = 0, kMaskSoftmax = 4;  // in words, from kSeq
  static constexpr int kTileList = (4 + 8 * 4) * 8;      // bytes, from kSeq
  static constexpr int kTileListBytes = 64 * kMaskWords * 2;
  static constexpr int kTileCount = kTileList + 2 * kTileListBytes;  // two ints
  static constexpr int kSeqBytes = PAGED ? (kPagedMaxBlocks + 2 * kPagedMaxSeqs + 1 + 1 + 16) * 4
                                         : SPARSE ? kTileCount + 2 * 4 : 0;
  static constexpr int kBar = (kSeq + kSeqBytes + 7) / 8 * 8;
  static constexpr int kBarQFull = 0;   // [tile]
  static constexpr int kBarQEmpty = 2;  // [tile]
  static constexpr int kBarKFull = 4;
  static constexpr int kBarKEmpty = kBarKFull + NS;
  static constexpr int kBarVFull = kBarKEmpty + NS;
  static constexpr int kBarVEmpty = kBarVFull + NS;
  static constexpr int kBarSFull = kBarVEmpty + NS;     // [tile]
  static constexpr int kBarPFull = kBarSFull + 2;       // [tile]
  static constexpr int kBarOFull = kBarPFull + 2;       // [tile]: O_t of the item is final
  static constexpr int kBarOFree = kBarOFull + 2;       // [tile]: the epilogue has read O_t
  static constexpr int kBarStatsFull = kBarOFree + 2;   // [tile][slot]
  static constexpr int kBarStatsEmpty = kBarStatsFull + 4;
  static constexpr int kBarMmaDone = kBarStatsEmpty + 4;
  static constexpr int kBarListFull = kBarMmaDone + 1;    // 2: block-sparse tile lists
  static constexpr int kBarListEmpty = kBarListFull + 2;  // 2
  static constexpr int kNumBars = kBarListEmpty + 2;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kBytes = kTmemSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack: the base is rounded up to 1024 B
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;        // O0 at 256, O1 at 256 + D
};

// One work item: 256 query rows [m*256, m*256+256) of head (b, h).  Query
// tile t (rows m*256 + 128t ...) sees the 128-key KV tiles j with
// lo[t] <= j < hi[t]; the item walks j over [jb, je), the union of both.
// Paged: b is the sequence, its new queries are packed rows q0 .. q0+n_q-1,
// query row r is token pos0 + r of a cache of n_kv tokens.
struct PrefillItem {
  int b, h, m;
  int lo0, hi0, lo1, hi1;  // tile 1 is empty (lo1 = hi1) when its rows lie past N
  int jb, je;
  int q0, n_q, n_kv, pos0;  // paged only
  // Block-sparse only: the KV tiles each query tile visits, as bits (tile j:
  // bit j % 64 of word j / 64), already limited to [lo, hi).
  uint64_t mk0[kMaskWords], mk1[kMaskWords];
  __device__ __forceinline__ int lo(int t) const { return t ? lo1 : lo0; }
  __device__ __forceinline__ int hi(int t) const { return t ? hi1 : hi0; }
  __device__ __forceinline__ bool active(int t, int j) const { return lo(t) <= j && j < hi(t); }
  __device__ __forceinline__ bool has(int t) const { return hi(t) > lo(t); }
};

// Bits [lo, hi) of a 64-bit word (0 <= lo, hi <= 64).
__device__ __forceinline__ uint64_t bit_range(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 64);
  if (hi <= lo) return 0ull;
  const uint64_t upto = hi == 64 ? ~0ull : ((1ull << hi) - 1ull);
  return upto & (~0ull << lo);
}

// Smallest set bit above j in a 4-word set, or 64 * kMaskWords if none.
__device__ __forceinline__ int next_bit(uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3, int j) {
  const int from = j + 1;
#pragma unroll
  for (int k = 0; k < kMaskWords; ++k) {
    uint64_t w = k == 0 ? w0 : k == 1 ? w1 : k == 2 ? w2 : w3;
    const int lo_bit = from - k * 64;
    if (lo_bit >= 64) continue;
    if (lo_bit > 0) w &= ~0ull << lo_bit;
    if (w) return k * 64 + __ffsll(static_cast<long long>(w)) - 1;
  }
  return 64 * kMaskWords;
}

// The same over four words in shared memory (read when needed).
__device__ __forceinline__ int next_bit_s(const volatile uint64_t* w, int j) {
  return next_bit(w[0], w[1], w[2], w[3], j);
}
__device__ __forceinline__ int next_bit_union_s(const volatile uint64_t* a, const volatile uint64_t* b, int j) {
  return next_bit(a[0] | b[0], a[1] | b[1], a[2] | b[2], a[3] | b[3], j);
}
__device__ __forceinline__ bool bit_s(const volatile uint64_t* w, int j) {
  return j >= 0 && j < 64 * kMaskWords && ((w[j >> 6] >> (j & 63)) & 1ull) != 0ull;
}
// Number of KV tiles query tile t of an item visits (block-sparse: its set's size).
template <bool SPARSE>
__device__ __forceinline__ int tile_count(const PrefillItem& it, int t) {
  if constexpr (SPARSE) {
    int n = 0;
#pragma unroll
    for (int k = 0; k < kMaskWords; ++k) n += __popcll(t ? it.mk1[k] : it.mk0[k]);
    return n;
  } else {
    return it.hi(t) - it.lo(t);
  }
}

// Sequence table of the paged kernels, in shared memory.
struct PagedSeqs {
  const int* blocks;   // [num_blocks]: query block (sequence s, block m) as s * 2048 + m, heaviest first
  const int* cu_q;     // [S + 1]
  const int* lens;     // [S]
  const int* nblocks;  // number of query blocks
};

// KV tiles the two query tiles of block m of a chunk visit (its work).
template <bool CAUSAL>
__device__ __forceinline__ int paged_block_tiles(int pos0, int n_q, int n_kv, int m) {
  const int last0 = CAUSAL ? min(pos0 + m * 256 + 127, n_kv - 1) : n_kv - 1;
  const int last1 = CAUSAL ? min(pos0 + m * 256 + 255, n_kv - 1) : n_kv - 1;
  return last0 / 128 + 1 + (m * 256 + 128 < n_q ? last1 / 128 + 1 : 0);
}

// Item idx = (block rank idx / Hq, head idx % Hq).
template <bool CAUSAL>
__device__ __forceinline__ bool paged_item(int idx, const PrefillParams& p, const PagedSeqs& sq,
                                           PrefillItem& it) {
  const int rank = idx / p.Hq;
  if (rank >= *sq.nblocks) return false;
  const int blk = sq.blocks[rank];
  const int s = blk >> 11;
  it.b = s;
  it.m = blk & 2047;
  it.h = idx - rank * p.Hq;
  it.q0 = sq.cu_q[s];
  it.n_q = sq.cu_q[s + 1] - it.q0;
  it.n_kv = sq.lens[s];
  it.pos0 = it.n_kv - it.n_q;
  {
    const int r0 = it.pos0 + it.m * 256;
    const int last_key = CAUSAL ? min(r0 + 127, it.n_kv - 1) : it.n_kv - 1;
    it.lo0 = 0;
    it.hi0 = last_key / 128 + 1;
  }
  if (it.m * 256 + 128 >= it.n_q) {
    it.lo1 = it.hi1 = 0;
  } else {
    const int r0 = it.pos0 + it.m * 256 + 128;
    const int last_key = CAUSAL ? min(r0 + 127, it.n_kv - 1) : it.n_kv - 1;
    it.lo1 = 0;
    it.hi1 = last_key / 128 + 1;
  }
  it.jb = 0;
  it.je = max(it.hi0, it.hi1);
  return true;
}

// The value, through a move the compiler cannot see into: what is derived
// from it is computed where it is used rather than hoisted and kept live.
__device__ __forceinline__ uint32_t opaque_u32(uint32_t x) {
  uint32_t y;
  asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Non-blocking: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Whether this CTA has an item in round `round` (prefill_item without the item).
template <bool PAGED>
__device__ __forceinline__ bool prefill_item_exists(int round, const PrefillParams& p, const PagedSeqs& sq) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const int idx = round * G + ((round & 1) ? (G - 1 - c) : c);
  if constexpr (PAGED) return idx / p.Hq < *sq.nblocks;
  return idx < p.num_items;
}

template <bool CAUSAL, bool WINDOW, bool PAGED = false, bool SPARSE = false>
__device__ __forceinline__ bool prefill_item(int round, const PrefillParams& p, PrefillItem& it,
                                             const PagedSeqs& sq = PagedSeqs{}) {
  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const int idx = round * G + ((round & 1) ? (G - 1 - c) : c);
  if constexpr (PAGED) return paged_item<CAUSAL>(idx, p, sq, it);
  if (idx >= p.num_items) return false;
  const int bh_count = p.B * p.Hq;
  const int rank = idx / bh_count;  // 0 = heaviest
  it.m = CAUSAL ? (p.num_m - 1 - rank) : rank;
  const int bh = idx % bh_count;
  it.b = bh / p.Hq;
  it.h = bh % p.Hq;
  // Tile t: rows r0 .. r0+127; visible keys from first (window) to last
  // (causal diagonal or N - 1).
  {
    const int r0 = it.m * 256;
    const int first_key = WINDOW ? max(0, r0 - p.window_left) : 0;
    const int last_key = CAUSAL ? min(r0 + 127, p.N - 1) : p.N - 1;
    it.lo0 = first_key / 128;
    it.hi0 = last_key / 128 + 1;
  }
  {
    const int r0 = it.m * 256 + 128;
    if (r0 >= p.N) {
      it.lo1 = it.hi1 = 0;
    } else {
      const int first_key = WINDOW ? max(0, r0 - p.window_left) : 0;
      const int last_key = CAUSAL ? min(r0 + 127, p.N - 1) : p.N - 1;
      it.lo1 = first_key / 128;
      it.hi1 = last_key / 128 + 1;
    }
  }
  it.jb = it.lo0;
  it.je = max(it.hi0, it.has(1) ? it.hi1 : 0);
  if constexpr (SPARSE) {
    const uint64_t* rows = p.block_mask + it.b * p.mask_b_stride + it.h * p.mask_h_stride;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint64_t* row = rows + static_cast<long long>(2 * it.m + t) * p.mask_words;
      const bool live = it.has(t);
#pragma unroll
      for (int k = 0; k < kMaskWords; ++k) {
        const uint64_t w = (live && k < p.mask_words) ? row[k] : 0ull;
        const uint64_t keep = w & bit_range(it.lo(t) - 64 * k, it.hi(t) - 64 * k);
        if (t) it.mk1[k] = keep; else it.mk0[k] = keep;
      }
    }
  }
  return true;
}

// Paged kernels: every CTA caches the sequence table in shared memory and
// lists the 256-row query blocks of all chunks, heaviest (most KV tiles)
// first, so the persistent CTAs, dealt items in that order, finish together.
// A sequence whose lengths are out of range gets no blocks and sets
// kErrPagedTable.  `scratch` is shared memory that is free until the main
// loop (the V ring): 2048 sort keys and S + 1 block offsets.  Called by all
// threads; ends with a barrier.
template <bool CAUSAL>
__device__ __forceinline__ void paged_seq_table(const PrefillParams& p, int* blocks, int* cuq, int* lens,
                                                int* nblocks, int* wsum, uint8_t* scratch) {
  const int S = p.num_seqs;
  const int tid = static_cast<int>(threadIdx.x);
  const int nthreads = static_cast<int>(blockDim.x);
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nw = nthreads >> 5;
  uint64_t* keys = reinterpret_cast<uint64_t*>(scratch);
  int* boff = reinterpret_cast<int*>(scratch + kPagedMaxBlocks * 8);  // [S + 1] first block of each sequence
  int v[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int sq = 2 * tid + e;
    v[e] = 0;
    if (sq < S) {
      const int a = p.cu_q[sq], b = p.cu_q[sq + 1], len = p.seq_lens[sq];
      cuq[sq] = a;
      lens[sq] = len;
      if (sq == S - 1) cuq[S] = b;
      const int nq = b - a;
      if (a < 0 || nq < 0 || b > p.total_q || nq > len || len > p.max_pages * p.page_size) {
        if (blockIdx.x == 0) atomicOr(&g_attn_device_error, kErrPagedTable);
      } else {
        v[e] = (nq + 255) / 256;
      }
    }
  }
  const int tot = v[0] + v[1];
  int x = tot;  // inclusive scan over the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) wsum[lane] = w;
  }
  __syncthreads();
  const int before = x - tot + (warp > 0 ? wsum[warp - 1] : 0);
  if (2 * tid < S) boff[2 * tid] = before;
  if (2 * tid + 1 < S) boff[2 * tid + 1] = before + v[0];
  int nb = wsum[nw - 1];
  if (nb > kPagedMaxBlocks) {  // only with inconsistent offsets (the host bounds the sum)
    if (blockIdx.x == 0 && tid == 0) atomicOr(&g_attn_device_error, kErrPagedTable);
    nb = 0;
  }
  if (tid == 0) {
    boff[S] = nb;
    *nblocks = nb;
  }
  __syncthreads();
  // Sort keys: work (KV tiles) high, then the block id s * 2048 + m inverted,
  // so equal work keeps sequence order; padding keys are 0 and sort last.
  int n = 1;
  while (n < nb) n <<= 1;
  for (int i = tid; i < n; i += nthreads) {
    uint64_t key = 0;
    if (i < nb) {
      int lo = 0, hi = S;  // boff[lo] <= i < boff[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (boff[mid] <= i) lo = mid; else hi = mid;
      }
      const int m = i - boff[lo];
      const int nq = cuq[lo + 1] - cuq[lo];
      const int w = paged_block_tiles<CAUSAL>(lens[lo] - nq, nq, lens[lo], m);
      key = (static_cast<uint64_t>(w) << 32) | (0xffffffffu - static_cast<uint32_t>(lo * 2048 + m));
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int k = 2; k <= n; k <<= 1) {  // bitonic sort, descending
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n; i += nthreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = keys[i], b = keys[ixj];
          if (((i & k) == 0) ? (a < b) : (a > b)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < nb; i += nthreads)
    blocks[i] = static_cast<int>(0xffffffffu - static_cast<uint32_t>(keys[i] & 0xffffffffu));
  fence_proxy_async_smem();  // TMA (async proxy) will overwrite the scratch keys
  __syncthreads();
}

// Register split per warpgroup (launch: 512 threads x 128 registers):
// softmax 2 x 184, epilogue 64, producer/MMA 80 -> 4 x 128 per lane slot.
__device__ __forceinline__ void reg_alloc_softmax() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 184;\n" ::: "memory");
}
__device__ __forceinline__ void reg_alloc_epilogue() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 64;\n" ::: "memory");
}
__device__ __forceinline__ void reg_alloc_control() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n" ::: "memory");
}

template <int D, bool CAUSAL, bool WINDOW, bool PAGED, bool FP8 = false, bool SPARSE = false, bool BIAS = false>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(!(PAGED && WINDOW), "the paged kernels have no window");
  static_assert(!(FP8 && (PAGED || WINDOW)), "the FP8 kernels are dense, without a window");
  static_assert(!(SPARSE && (PAGED || WINDOW || FP8)), "the block-sparse kernels are dense bf16");
  static_assert(!(BIAS && (PAGED || WINDOW || FP8 || SPARSE)), "the additive-M kernels are dense bf16");
  using L = PrefillLayout<D, PAGED, FP8, SPARSE>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8u * static_cast<uint32_t>(i); };
  float* stats = reinterpret_cast<float*>(smem + L::kStats);
  // Block-sparse mask words (SPARSE only), see PrefillLayout.
  volatile uint64_t* const mask_smem = reinterpret_cast<volatile uint64_t*>(smem + L::kSeq);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  PagedSeqs sq{};
  if constexpr (PAGED) {
    int* blocks = reinterpret_cast<int*>(smem + L::kSeq);
    int* cuq = blocks + kPagedMaxBlocks;
    int* lens = cuq + kPagedMaxSeqs + 1;
    int* nblocks = lens + kPagedMaxSeqs;
    paged_seq_table<CAUSAL>(p, blocks, cuq, lens, nblocks, nblocks + 1, smem + L::kV);
    sq = PagedSeqs{blocks, cuq, lens, nblocks};
  }

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kBarQFull + t), 1);
      mbar_init(bar(L::kBarQEmpty + t), 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kBarSFull + t), 1);
      mbar_init(bar(L::kBarPFull + t), 128);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kBarOFull + t), 1);
      mbar_init(bar(L::kBarOFree + t), 128);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(L::kBarStatsFull + i), 128);
      mbar_init(bar(L::kBarStatsEmpty + i), 128);
    }
    mbar_init(bar(L::kBarMmaDone), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::kBarListFull + i), 1);
      mbar_init(bar(L::kBarListEmpty + i), 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 13) {
    tmem_alloc(base + L::kTmemSlot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  if (wg == 3) {
    reg_alloc_control();
    if (warp == 12) {
      // ---------------------------------------------------------- producer
      // Lane 0 waits and issues the copies; the paged kernels also use the
      // other lanes for block-table lookups and the partly used last page.
      int kv_it = 0, k_issued = 0, v_issued = 0;
      int q_issued[2] = {0, 0};  // loads of Q tile t
      bool ok = true;
      PrefillItem it{};
      // Paged: the tile whose pages t_row / t_valid describe (lane b: box b),
      // and a 32-entry window of the item's block-table row (lane l: entry
      // win_base + l) with the next 32 entries prefetched in win_next.
      int tile_j = -1, t_row = 0, t_valid = 0;
      int win_base = -(1 << 30), win_page = -1, win_next = -1;
      bool have_next = false;
      auto wait0 = [&](uint32_t b, uint32_t parity, unsigned int code) -> bool {
        int r = 1;
        if (lane == 0) r = mbar_wait(b, parity, code) ? 1 : 0;
        return __shfl_sync(0xffffffffu, r, 0) != 0;
      };
      // Keys 128j .. 128j+127 of K or V into the stage at dst.
      auto load_tile = [&](const CUtensorMap* map, const __nv_bfloat16* pool, uint32_t dst, uint32_t full, int j,
                           int kz) {
        if constexpr (!PAGED) {
          if (lane == 0) {
            mbar_arrive_expect_tx(full, L::kTileBytes);
            for (int c = 0; c < L::kBoxes; ++c)
              tma_load_3d(dst + c * L::kBoxBytes, map, full, c * L::kBoxCols, j * 128, kz);
          }
        } else {
          // Box b (lane b) holds keys 128j + b*pb ...: a page (or a 128-key
          // part of one) found through the block table.  Boxes wholly past the
          // sequence start outside the pool, so TMA fills them with zeros.
          // K and V of a tile share their pages: resolved once, for K.
          const int pb = p.page_box;
          const int nbox = 128 / pb;
          if (tile_j != j) {
            tile_j = j;
            const int lp_first = (j * 128) / p.page_size;
            const int lp_last = (j * 128 + 127) / p.page_size;
            if (lp_first < win_base || lp_last >= win_base + 32) {
              // Lane l holds the table entry of logical page win_base + l; the
              // next 32 entries are fetched ahead, while this window is used.
              const int* trow = p.block_table + static_cast<size_t>(it.b) * p.max_pages;
              const bool follow = have_next && lp_first == win_base + 32;
              win_base = lp_first;
              win_page = follow ? win_next : (win_base + lane < p.max_pages ? trow[win_base + lane] : -1);
              win_next = win_base + 32 + lane < p.max_pages ? trow[win_base + 32 + lane] : -1;
              have_next = true;
            }
            const int pos = j * 128 + lane * pb;
            const int pg_raw = __shfl_sync(0xffffffffu, win_page, (pos / p.page_size - win_base) & 31);
            t_row = p.num_pages * p.page_size;
            t_valid = pb;
            if (lane < nbox && pos < it.n_kv) {
              int pg = pg_raw;
              if (pg < 0 || pg >= p.num_pages) {
                atomicOr(&g_attn_device_error, kErrPagedTable);
                pg = 0;  // keep every copy inside the pool; the result is flagged invalid
              }
              t_row = pg * p.page_size + pos % p.page_size;
              t_valid = min(pb, it.n_kv - pos);
            }
          }
          const int row = t_row;
          const int valid = t_valid;
          // The box with the sequence's last token, when only part of it is
          // used, comes through 16-byte cp.async copies instead: the slots past
          // the end may hold anything (even NaN), so they are filled with
          // zeros (source size 0).  Each lane's copies hold the stage's phase
          // open until they land.
          const unsigned part = __ballot_sync(0xffffffffu, lane < nbox && valid < pb);
          if (part != 0u) {
            const int b = __ffs(part) - 1;
            const int prow = __shfl_sync(0xffffffffu, row, b);
            const int pval = __shfl_sync(0xffffffffu, valid, b);
            constexpr int kChunks = (D / 64) * 8;  // 16-byte chunks per row
            for (int idx = lane; idx < pb * kChunks; idx += 32) {
              const int r = idx / kChunks;
              const int c = (idx % kChunks) / 8;   // 64-column half
              const int ch = idx % 8;              // chunk within the 128-byte row
              const int tr = b * pb + r;           // row within the tile
              const bool in = r < pval;
              const __nv_bfloat16* src =
                  in ? pool + ((static_cast<size_t>(prow + r) * p.Hkv + kz) * D + c * 64 + ch * 8) : pool;
              cp_async_16(dst + static_cast<uint32_t>(c * L::kBoxBytes + tr * 128 + ((ch ^ (tr & 7)) << 4)), src,
                          in ? 16u : 0u);
            }
            cp_async_mbar_arrive(full);
          }
          __syncwarp();
          const int ntma = nbox - (part != 0u ? 1 : 0);
          if (lane == 0) {
            if (ntma > 0)
              mbar_arrive_expect_tx(full, static_cast<uint32_t>(ntma * pb * 128 * (D / 64)));
            else
              mbar_arrive(full);
          }
          // Lane b issues box b: a one-thread loop over the boxes (a shuffle
          // and two copies each) made the producer the bottleneck for
          // 16-token pages.
          __syncwarp();
          if (lane < nbox && ((part >> lane) & 1u) == 0u)
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(dst + static_cast<uint32_t>(c * L::kBoxBytes + lane * pb * 128), map, full, c * 64, row,
                          kz);
        }
      };
      auto load_k = [&](int j, int kz) -> bool {
        const int st = kv_it % NS;
        const uint32_t round = static_cast<uint32_t>(kv_it / NS);
        if (round > 0 && !wait0(bar(L::kBarKEmpty + st), (round - 1) & 1u, kErrWaitKEmpty)) return false;
        load_tile(&tm_k, p.k_pool, base + L::kK + st * L::kTileBytes, bar(L::kBarKFull + st), j, kz);
        ++k_issued;
        return true;
      };
      auto load_v = [&](int j, int kz) -> bool {
        const int st = kv_it % NS;
        const uint32_t round = static_cast<uint32_t>(kv_it / NS);
        if (round > 0 && !wait0(bar(L::kBarVEmpty + st), (round - 1) & 1u, kErrWaitVEmpty)) return false;
        load_tile(&tm_v, p.v_pool, base + L::kV + st * L::kTileBytes, bar(L::kBarVFull + st), j, kz);
        ++v_issued;
        return true;
      };
      for (int r = 0; ok && prefill_item<CAUSAL, WINDOW, PAGED, SPARSE>(r, p, it, sq); ++r) {
        // Q rows: dense (d, row, b*Hq + h); paged (d, packed token, h).
        const int qz = PAGED ? it.h : it.b * p.Hq + it.h;
        const int qrow = (PAGED ? it.q0 : 0) + it.m * 256;
        // GQA: consecutive query heads share a KV head
        const int kz = (PAGED ? 0 : it.b * p.Hkv) + it.h / p.group;
        tile_j = -1;  // a new item: its own sequence, pages and table row
        win_base = -(1 << 30);
        have_next = false;
        // Block-sparse: the item's union of sets, in shared memory for the warp.
        volatile uint64_t* const mu = mask_smem + L::kMaskProd;
        if constexpr (SPARSE) {
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int k = 0; k < kMaskWords; ++k) mu[k] = it.mk0[k] | it.mk1[k];
          }
          __syncwarp();
        }
        auto unext = [&](int j) { return SPARSE ? min(next_bit_s(mu, j), it.je) : j + 1; };
        const int j0 = SPARSE ? unext(it.jb - 1) : it.jb;
        if (j0 >= it.je) continue;  // block-sparse: every tile of the item masked, nothing to load
        // The item's first K tile first: it can land while the previous item
        // still holds Q.
        if (!(ok = load_k(j0, kz))) break;
        // Q0 and Q1 are released separately, each after its query tile's last
        // S of the previous item, so Q0 can arrive while Q1 is still in use.
        for (int t = 0; t < 2; ++t) {
          if (t == 1 && !it.has(1)) break;
          if (q_issued[t] > 0 &&
              !(ok = wait0(bar(L::kBarQEmpty + t), static_cast<uint32_t>(q_issued[t] - 1) & 1u, kErrWaitQ)))
            break;
          if (lane == 0) {
            mbar_arrive_expect_tx(bar(L::kBarQFull + t), L::kTileBytes);
            for (int c = 0; c < L::kBoxes; ++c)
              tma_load_3d(base + (t ? L::kQ1 : L::kQ0) + c * L::kBoxBytes, &tm_q, bar(L::kBarQFull + t),
                          c * L::kBoxCols, qrow + 128 * t, qz);
          }
          ++q_issued[t];
        }
        if (!ok) break;
        if (!(ok = load_v(j0, kz))) break;
        ++kv_it;
        for (int j = unext(j0); j < it.je; j = unext(j), ++kv_it) {
          if (!(ok = load_k(j, kz))) break;
          if (!(ok = load_v(j, kz))) break;
        }
      }
      // Every copy this warp started must land before the CTA may exit.
      if (lane == 0) {
        for (int t = 0; t < 2; ++t)
          if (q_issued[t] > 0)
            mbar_wait(bar(L::kBarQFull + t), static_cast<uint32_t>(q_issued[t] - 1) & 1u, kErrWaitDrain);
        for (int j = max(0, k_issued - NS); j < k_issued; ++j)
          mbar_wait(bar(L::kBarKFull + j % NS), static_cast<uint32_t>(j / NS) & 1u, kErrWaitDrain);
        for (int j = max(0, v_issued - NS); j < v_issued; ++j)
          mbar_wait(bar(L::kBarVFull + j % NS), static_cast<uint32_t>(j / NS) & 1u, kErrWaitDrain);
      }
      __syncwarp();
    } else if (warp == 13 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk =
          FP8 ? make_idesc_e4m3(128, 128, false, false) : make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = FP8 ? make_idesc_e4m3(128, D, false, true) : make_idesc_bf16(128, D, false, true);
      // The next item's first S0 is issued during the current item's last
      // tile (below), so query tile 0 starts the next item while query tile 1
      // finishes this one.  Windowed items are long and equal: they skip it.
      constexpr bool kEarlyS0 = !WINDOW;
      // Every MMA takes 32 bytes of its K dimension: 16 bf16 or 32 e4m3.
      constexpr int kSSteps = D * L::kElemBytes / 32;     // S = Q K^T over the head dim
      constexpr int kPvKeys = 32 / L::kElemBytes;         // keys per P V step
      constexpr int kPvSteps = 128 / kPvKeys;
      int kv_it = 0;
      uint32_t p_cnt[2] = {0u, 0u};
      uint32_t o_cnt[2] = {0u, 0u};  // items whose O_t has been completed
      bool ok = true;
      auto issue_s = [&](int t, int st, bool opaque = false) {
        // Addresses through an opaque move make a call site derive its
        // descriptors in place instead of holding them across the loops: the
        // early S0's site always (it would otherwise widen the hoisted set
        // past the MMA thread's registers), every site in the FP8 kernel.
        const bool op = FP8 || opaque;
        const uint32_t q_addr = op ? opaque_u32(base + (t ? L::kQ1 : L::kQ0)) : base + (t ? L::kQ1 : L::kQ0);
        const uint32_t k_addr = op ? opaque_u32(base + L::kK + st * L::kTileBytes) : base + L::kK + st * L::kTileBytes;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(t) * 128u;
#pragma unroll
        for (int kk = 0; kk < kSSteps; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * L::kBoxBytes + (kk & 3) * 32);
          if constexpr (FP8)
            mma_f8_ss_lo(d_tmem, sdesc_sw128_lo<16>(q_addr + off), sdesc_sw128_lo<16>(k_addr + off), idesc_qk,
                         kk > 0 ? 1u : 0u);
          else
            mma_bf16_ss_lo(d_tmem, sdesc_sw128_lo<16>(q_addr + off), sdesc_sw128_lo<16>(k_addr + off), idesc_qk,
                           kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::kBarSFull + t));
      };
      auto issue_pv = [&](int t, int st, bool accumulate) {
        const uint32_t v_addr = FP8 ? opaque_u32(base + L::kV + st * L::kTileBytes) : base + L::kV + st * L::kTileBytes;
        const uint32_t p_tmem = tmem + static_cast<uint32_t>(t) * 128u;
        const uint32_t o_tmem = tmem + L::kColO + static_cast<uint32_t>(t * D);
#pragma unroll
        for (int kk = 0; kk < kPvSteps; ++kk) {
          // P: 32 bytes of a row per step = 8 TMEM columns; V: kPvKeys rows of 128 bytes.
          const uint32_t vdesc = sdesc_sw128_lo<L::kBoxBytes>(v_addr + kk * kPvKeys * 128);
          if constexpr (FP8)
            mma_f8_ts_lo(o_tmem, p_tmem + kk * 8, vdesc, idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
          else
            mma_bf16_ts_lo(o_tmem, p_tmem + kk * 8, vdesc, idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      PrefillItem it;
      if constexpr (SPARSE) {
        // Block-sparse: each query tile visits an arbitrary set of KV tiles;
        // the item walks their union.
        uint32_t q_cnt[2] = {0u, 0u};  // loads of Q tile t waited for (fully masked items load none)
        for (int r = 0; ok; ++r) {
          // The item's tile list, from the lister warp (length -1: no items left).
          const int buf = r & 1;
          if (!(ok = mbar_wait(bar(L::kBarListFull + buf), static_cast<uint32_t>(r >> 1) & 1u, kErrWaitList))) break;
          const volatile uint16_t* const tl =
              reinterpret_cast<const volatile uint16_t*>(smem + L::kSeq + L::kTileList + buf * L::kTileListBytes);
          const int n_raw = reinterpret_cast<const volatile int*>(smem + L::kSeq + L::kTileCount)[buf];
          if (n_raw < 0) break;
          const int n_u = n_raw & 0xffff;
          const bool has1 = (n_raw >> 30) & 1;
          if (n_u == 0) {  // nothing to compute (the epilogue writes zeros)
            mbar_arrive(bar(L::kBarListEmpty + buf));
            continue;
          }
          auto on = [&](int t, int e) { return ((e >> (8 + t)) & 1) != 0; };
          if (!(ok = mbar_wait(bar(L::kBarQFull + 0), q_cnt[0] & 1u, kErrWaitQ))) break;
          ++q_cnt[0];
          if (has1) {
            if (!(ok = mbar_wait(bar(L::kBarQFull + 1), q_cnt[1] & 1u, kErrWaitQ))) break;
            ++q_cnt[1];
          }
          {
            const int st = kv_it % NS;
            if (!(ok = mbar_wait(bar(L::kBarKFull + st), static_cast<uint32_t>(kv_it / NS) & 1u, kErrWaitKFull)))
              break;
            tc_fence_after();
            if (on(0, tl[0])) issue_s(0, st);
            if (on(1, tl[0])) issue_s(1, st);
            mma_commit(bar(L::kBarKEmpty + st));
            if (n_u == 1) {  // last S of the item
              mma_commit(bar(L::kBarQEmpty + 0));
              if (has1) mma_commit(bar(L::kBarQEmpty + 1));
            }
          }
          // First and last KV tile of each query tile: where O_t starts (after
          // the epilogue released it) and where it is final.
          auto first_of = [&](int t, int e) { return ((e >> (10 + t)) & 1) != 0; };
          auto last_of = [&](int t, int e) { return ((e >> (12 + t)) & 1) != 0; };
          int u = 0;  // position among the item's tiles (K/V ring slot kv_it + u)
          for (; u < n_u && ok; ++u) {
            const int e = tl[u];                        // this tile
            const bool more = u + 1 < n_u;
            const int en = more ? tl[u + 1] : 0;        // the next one
            const int g = kv_it + u;
            const int st = g % NS, st1 = (g + 1) % NS;
            const uint32_t ph = static_cast<uint32_t>(g / NS) & 1u, ph1 = static_cast<uint32_t>((g + 1) / NS) & 1u;
            bool v_ready = false, k_ready = false;
            if (on(0, e)) {
              const uint32_t pph = p_cnt[0]++ & 1u;
              if (!(ok = mbar_wait(bar(L::kBarPFull + 0), pph, kErrWaitPFull))) break;
              if (first_of(0, e) && o_cnt[0] > 0 &&
                  !(ok = mbar_wait(bar(L::kBarOFree + 0), (o_cnt[0] - 1u) & 1u, kErrWaitODone)))
                break;
              if (!(ok = mbar_wait(bar(L::kBarVFull + st), ph, kErrWaitVFull))) break;
              v_ready = true;
              tc_fence_after();
              issue_pv(0, st, !first_of(0, e));
              if (last_of(0, e)) {
                mma_commit(bar(L::kBarOFull + 0));  // O0 of this item is final once this lands
                ++o_cnt[0];
              }
            }
            if (more && on(0, en)) {
              // Q0's next S.  P0, which S0 overwrites, went into a P V already
              // issued (this tile's or an earlier one's).
              if (!(ok = mbar_wait(bar(L::kBarKFull + st1), ph1, kErrWaitKFull))) break;
              k_ready = true;
              tc_fence_after();
              issue_s(0, st1);
            }
            if (on(1, e)) {
              const uint32_t pph = p_cnt[1]++ & 1u;
              if (!(ok = mbar_wait(bar(L::kBarPFull + 1), pph, kErrWaitPFull))) break;
              if (first_of(1, e) && o_cnt[1] > 0 &&
                  !(ok = mbar_wait(bar(L::kBarOFree + 1), (o_cnt[1] - 1u) & 1u, kErrWaitODone)))
                break;
              if (!v_ready && !(ok = mbar_wait(bar(L::kBarVFull + st), ph, kErrWaitVFull))) break;
              tc_fence_after();
              issue_pv(1, st, !first_of(1, e));
              if (last_of(1, e)) {
                mma_commit(bar(L::kBarOFull + 1));
                ++o_cnt[1];
              }
            }
            if (more && on(1, en)) {
              // Q1's next S; also its first one when its range starts at jn.
              if (!k_ready && !(ok = mbar_wait(bar(L::kBarKFull + st1), ph1, kErrWaitKFull))) break;
              tc_fence_after();
              issue_s(1, st1);
            }
            mma_commit(bar(L::kBarVEmpty + st));
            if (more) mma_commit(bar(L::kBarKEmpty + st1));
            if (u + 2 == n_u) {  // the item's last S MMAs were just issued
              mma_commit(bar(L::kBarQEmpty + 0));
              if (has1) mma_commit(bar(L::kBarQEmpty + 1));
            }
          }
          if (!ok) break;
          kv_it += u;
          mbar_arrive(bar(L::kBarListEmpty + buf));  // the list may be rewritten
        }
      } else {
        // Dense: query tile t visits the contiguous range [lo(t), hi(t)).
        uint32_t q_cnt[2] = {0u, 0u};  // loads of Q tile t waited for
        bool s0_early = false;         // this item's first S0 was issued during the previous item
        for (int r = 0; ok && prefill_item<CAUSAL, WINDOW, PAGED, SPARSE>(r, p, it, sq); ++r) {
          // Every item's query tile 0 starts at the item's first KV tile, so
          // only the next item's existence matters for the early S0 below.
          const bool have_nx = kEarlyS0 && prefill_item_exists<PAGED>(r + 1, p, sq);
          const int nkv = it.je - it.jb;
          {
            const int st = kv_it % NS;
            if (!s0_early) {
              if (!(ok = mbar_wait(bar(L::kBarQFull + 0), q_cnt[0] & 1u, kErrWaitQ))) break;
              ++q_cnt[0];
              if (!(ok = mbar_wait(bar(L::kBarKFull + st), static_cast<uint32_t>(kv_it / NS) & 1u, kErrWaitKFull)))
                break;
              tc_fence_after();
              if (it.active(0, it.jb)) issue_s(0, st);
            }
            s0_early = false;
            if (it.has(1)) {
              if (!(ok = mbar_wait(bar(L::kBarQFull + 1), q_cnt[1] & 1u, kErrWaitQ))) break;
              ++q_cnt[1];
              tc_fence_after();
              if (it.active(1, it.jb)) issue_s(1, st);
            }
            mma_commit(bar(L::kBarKEmpty + st));
            // A query tile's Q may be replaced once its last S is issued.
            if (it.hi0 - 1 == it.jb) mma_commit(bar(L::kBarQEmpty + 0));
            if (it.has(1) && it.hi1 - 1 == it.jb) mma_commit(bar(L::kBarQEmpty + 1));
          }
          for (int j = it.jb; j < it.je && ok; ++j) {
            const int g = kv_it + (j - it.jb);
            const int st = g % NS, st1 = (g + 1) % NS;
            const uint32_t ph = static_cast<uint32_t>(g / NS) & 1u, ph1 = static_cast<uint32_t>((g + 1) / NS) & 1u;
            bool v_ready = false, k_ready = false;
            if (it.active(0, j)) {
              const uint32_t pph = p_cnt[0]++ & 1u;
              if (!(ok = mbar_wait(bar(L::kBarPFull + 0), pph, kErrWaitPFull))) break;
              if (j == it.lo0 && o_cnt[0] > 0 &&
                  !(ok = mbar_wait(bar(L::kBarOFree + 0), (o_cnt[0] - 1u) & 1u, kErrWaitODone)))
                break;
              if (!(ok = mbar_wait(bar(L::kBarVFull + st), ph, kErrWaitVFull))) break;
              v_ready = true;
              tc_fence_after();
              issue_pv(0, st, j > it.lo0);
              if (j + 1 == it.hi0) {
                mma_commit(bar(L::kBarOFull + 0));  // O0 of this item is final once this lands
                ++o_cnt[0];
              }
              if (it.active(0, j + 1)) {
                if (!(ok = mbar_wait(bar(L::kBarKFull + st1), ph1, kErrWaitKFull))) break;
                k_ready = true;
                tc_fence_after();
                issue_s(0, st1);
                if (j + 2 == it.hi0) mma_commit(bar(L::kBarQEmpty + 0));  // Q0's last S
              }
            }
            if (it.active(1, j)) {
              const uint32_t pph = p_cnt[1]++ & 1u;
              if (!(ok = mbar_wait(bar(L::kBarPFull + 1), pph, kErrWaitPFull))) break;
              if (j == it.lo1 && o_cnt[1] > 0 &&
                  !(ok = mbar_wait(bar(L::kBarOFree + 1), (o_cnt[1] - 1u) & 1u, kErrWaitODone)))
                break;
              if (!v_ready && !(ok = mbar_wait(bar(L::kBarVFull + st), ph, kErrWaitVFull))) break;
              tc_fence_after();
              issue_pv(1, st, j > it.lo1);
              if (j + 1 == it.hi1) {
                mma_commit(bar(L::kBarOFull + 1));
                ++o_cnt[1];
              }
            }
            if (it.active(1, j + 1)) {
              // Q1's next S; also its first one when its window starts at j + 1.
              if (!k_ready && !(ok = mbar_wait(bar(L::kBarKFull + st1), ph1, kErrWaitKFull))) break;
              tc_fence_after();
              issue_s(1, st1);
              if (j + 2 == it.hi1) mma_commit(bar(L::kBarQEmpty + 1));  // Q1's last S
            }
            mma_commit(bar(L::kBarVEmpty + st));
            if (j + 1 < it.je) mma_commit(bar(L::kBarKEmpty + st1));
            if (kEarlyS0 && j + 1 == it.hi0 && have_nx) {
              // Q0's work of this item is all issued (its last P V just now, so
              // P0 is consumed).  If the next item's Q0 and first K tile have
              // already landed, issue its first S0 now: query tile 0 then
              // starts the next item while query tile 1 finishes this one.
              // Only tests: nothing here waits.
              const int gn = kv_it + nkv;
              const int stn = gn % NS;
              if (mbar_test(bar(L::kBarQFull + 0), q_cnt[0] & 1u) &&
                  mbar_test(bar(L::kBarKFull + stn), static_cast<uint32_t>(gn / NS) & 1u)) {
                ++q_cnt[0];
                tc_fence_after();
                issue_s(0, stn, true);
                s0_early = true;
              }
            }
          }
          if (!ok) break;
          kv_it += nkv;
        }
      }
      // All issued MMAs must finish before tensor memory is released.
      mma_commit(bar(L::kBarMmaDone));
      mbar_wait(bar(L::kBarMmaDone), 0, kErrWaitMmaDone);
    } else if (SPARSE && warp == 14) {
      // ---------------------------------------------------------- tile lister
      // Block-sparse: lists each item's tiles in order, one item ahead of the
      // MMA thread, one 16-bit entry per tile: tile index (bits 0-7), visited
      // by query tile 0 / 1 (bits 8, 9), first for it (10, 11), last for it
      // (12, 13).  Lane l takes tiles 8l .. 8l+7 of the item's mask words
      // (already limited to the tiles each query tile can see) and writes them
      // at the prefix sum of the lower lanes' counts.
      PrefillItem it;
      for (int r = 0;; ++r) {
        const bool have = prefill_item<CAUSAL, WINDOW, PAGED, SPARSE>(r, p, it, sq);
        const int buf = r & 1;
        if (r >= 2) {  // the MMA thread is done with the list of item r - 2
          int okw = 1;
          if (lane == 0)
            okw = mbar_wait(bar(L::kBarListEmpty + buf), static_cast<uint32_t>((r >> 1) - 1) & 1u, kErrWaitList);
          if (__shfl_sync(0xffffffffu, okw, 0) == 0) break;
        }
        volatile uint16_t* const tl =
            reinterpret_cast<volatile uint16_t*>(smem + L::kSeq + L::kTileList + buf * L::kTileListBytes);
        int n_u = -1;
        if (have) {
          static_assert(kMaskWords == 4, "one mask word per 8 lanes");
          const int kw = lane >> 3;
          const uint64_t w0 = kw == 0 ? it.mk0[0] : kw == 1 ? it.mk0[1] : kw == 2 ? it.mk0[2] : it.mk0[3];
          const uint64_t w1 = kw == 0 ? it.mk1[0] : kw == 1 ? it.mk1[1] : kw == 2 ? it.mk1[2] : it.mk1[3];
          const int sh = (lane & 7) * 8;
          const uint32_t b0 = static_cast<uint32_t>(w0 >> sh) & 0xffu;
          const uint32_t b1 = static_cast<uint32_t>(w1 >> sh) & 0xffu;
          const uint32_t ub = b0 | b1;
          int incl = __popc(ub);
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          n_u = __shfl_sync(0xffffffffu, incl, 31);
          const uint32_t any0 = __ballot_sync(0xffffffffu, b0 != 0u);
          const uint32_t any1 = __ballot_sync(0xffffffffu, b1 != 0u);
          // This lane's bit (if any) that is the first / last tile of set 0 / 1.
          const int f0 = (lane == __ffs(any0) - 1) ? __ffs(b0) - 1 : -1;
          const int f1 = (lane == __ffs(any1) - 1) ? __ffs(b1) - 1 : -1;
          const int l0 = (any0 != 0u && lane == 31 - __clz(any0)) ? 31 - __clz(b0) : -1;
          const int l1 = (any1 != 0u && lane == 31 - __clz(any1)) ? 31 - __clz(b1) : -1;
          int pos = incl - __popc(ub);
          for (uint32_t rest = ub; rest != 0u; rest &= rest - 1u) {
            const int b = __ffs(rest) - 1;
            int e = (8 * lane + b) | static_cast<int>(((b0 >> b) & 1u) << 8) | static_cast<int>(((b1 >> b) & 1u) << 9);
            if (b == f0) e |= 1 << 10;
            if (b == f1) e |= 1 << 11;
            if (b == l0) e |= 1 << 12;
            if (b == l1) e |= 1 << 13;
            tl[pos++] = static_cast<uint16_t>(e);
          }
        }
        // Length, and bit 30: the item has a second query tile (its Q1 is loaded).
        if (lane == 0)
          reinterpret_cast<volatile int*>(smem + L::kSeq + L::kTileCount)[buf] =
              n_u < 0 ? n_u : (n_u | (it.has(1) ? 1 << 30 : 0));
        __threadfence_block();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::kBarListFull + buf));  // release: the entries above are visible
        if (!have) break;
      }
    }
    __syncwarp();
  } else if (wg == 2) {
    // ------------------------------------------------------------ epilogue
    reg_alloc_epilogue();
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    uint32_t st_cnt[2] = {0u, 0u};  // items whose tile t this warpgroup has written out
    bool ok = true;
    PrefillItem it;
    for (int r = 0; ok && prefill_item<CAUSAL, WINDOW, PAGED, SPARSE>(r, p, it, sq); ++r) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!it.has(t)) continue;
        if constexpr (SPARSE) {
          if (tile_count<SPARSE>(it, t) == 0) {
            // Every KV tile of this query tile is masked: its rows see no key,
            // O = 0 and LSE = -inf, with nothing computed to wait for.
            const int grow = it.m * 256 + t * 128 + row;
            if (grow < p.N) {
              const size_t row_index = static_cast<size_t>(it.b * p.Hq + it.h) * p.N + grow;
              uint4* dst = reinterpret_cast<uint4*>(p.o + row_index * D);
#pragma unroll
              for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
              p.lse[row_index] = -INFINITY;
            }
            continue;
          }
        }
        const uint32_t n = st_cnt[t];
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarOFull + t), n & 1u, kErrWaitODone));
        if (!ok) break;
        const uint32_t slot = n & 1u;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarStatsFull + 2 * t + slot), (n >> 1) & 1u,
                                               kErrWaitSFull));
        if (!ok) break;
        tc_fence_after();
        const float* sp = stats + ((t * 2 + slot) * 2) * 128;
        const float m_used = sp[row];
        const float l_sum = sp[128 + row];
        mbar_arrive(bar(L::kBarStatsEmpty + 2 * t + slot));
        ++st_cnt[t];
        const int grow = it.m * 256 + t * 128 + row;  // query row of the head (paged: of the sequence's chunk)
        // FP8: l carries P's 2^8 as O does.  Additive M can leave a row with
        // no finite score (l = 0): O = 0, LSE = -inf.
        const float inv_l = (BIAS && l_sum == 0.f) ? 0.f : (FP8 ? p.o_scale : 1.f) / l_sum;
        // O row / LSE index: dense [B, Hq, N, D] / [B, Hq, N]; paged by token, [total_q, Hq, D] / [total_q, Hq].
        const bool valid = grow < (PAGED ? it.n_q : p.N);
        const size_t row_index = PAGED ? (static_cast<size_t>(it.q0) + grow) * p.Hq + it.h
                                       : static_cast<size_t>(it.b * p.Hq + it.h) * p.N + grow;
        __nv_bfloat16* orow = p.o + row_index * D;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld_x32_wait(lane_addr + L::kColO + static_cast<uint32_t>(t * D + c), o);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
            dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
          }
        }
        if (valid)
          p.lse[row_index] = (BIAS && l_sum == 0.f) ? -INFINITY
                                                    : (m_used + log2f(l_sum) - (FP8 ? kFp8PLog2 : 0.f)) * kLn2;
        tc_fence_before();
        mbar_arrive(bar(L::kBarOFree + t));
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (tile t = wg)
    reg_alloc_softmax();
    const int t = wg;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_addr + static_cast<uint32_t>(t) * 128u;
    const uint32_t o_addr = lane_addr + L::kColO + static_cast<uint32_t>(t * D);
    const float sl2 = p.scale_log2;
    uint32_t s_cnt = 0, st_cnt = 0;
    bool ok = true;
    PrefillItem it;
    for (int r = 0; ok && prefill_item<CAUSAL, WINDOW, PAGED, SPARSE>(r, p, it, sq); ++r) {
      // Block-sparse: this query tile's set, in this warp's shared-memory slot.
      volatile uint64_t* const mw = mask_smem + L::kMaskSoftmax + warp * kMaskWords;
      if constexpr (SPARSE) {
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < kMaskWords; ++k) mw[k] = t ? it.mk1[k] : it.mk0[k];
        }
        __syncwarp();
      }
      const int lo_t = SPARSE ? next_bit_s(mw, -1) : it.lo(t);
      // KV tiles it visits (>= 0); block-sparse: 1 when the set is not empty
      // (its loop ends on the set's last tile instead).
      const int n_t = SPARSE ? (lo_t < 64 * kMaskWords ? 1 : 0) : it.hi(t) - lo_t;
      if (n_t == 0) continue;
      // Position (key index) of this tile's first query row; paged chunks
      // start at the sequence's cached length.
      const int row0 = (PAGED ? it.pos0 : 0) + it.m * 256 + t * 128;
      const int grow = row0 + row;
      const int n_kv = PAGED ? it.n_kv : p.N;
      float m_used = -INFINITY;  // running max in scaled log2 units
      float l_sum = 0.f;
      int j_set = lo_t - 1;  // block-sparse: the previous tile of this query tile's set
      for (int jj = 0; SPARSE ? next_bit_s(mw, j_set) < 64 * kMaskWords : jj < n_t; ++jj) {
        const int j = SPARSE ? (j_set = next_bit_s(mw, j_set)) : lo_t + jj;
        const int kv0 = j * 128;
        // Additive M: this row's 128 values of the tile, loaded (bf16, 16-byte
        // vectors) while the MMA computes S.  Vectors past N and rows past N
        // read nothing.
        uint4 mb[BIAS ? 16 : 1];
        if constexpr (BIAS) {
          const __nv_bfloat16* brow = p.bias + it.b * p.bias_b_stride + it.h * p.bias_h_stride +
                                      static_cast<long long>(grow) * p.bias_row_stride + kv0;
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            mb[v] = make_uint4(0u, 0u, 0u, 0u);
            if (grow < p.N && kv0 + 8 * v < p.N) mb[v] = __ldg(reinterpret_cast<const uint4*>(brow) + v);
          }
          // The next tile's 256 bytes of this row into L2 (two lines), one step
          // before they are loaded; only bytes that load reads.  (Two or three
          // steps ahead measured slower, and bulk prefetches from the producer
          // warp clogged the copy engine that brings K and V.)
          if (!SPARSE && grow < p.N && jj + 1 < n_t) {
            const int kv1 = kv0 + 128;
            const char* nxt = reinterpret_cast<const char*>(brow + 128);
            if (kv1 < p.N) prefetch_l2(nxt);
            if (kv1 + 64 < p.N) prefetch_l2(nxt + 128);
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarSFull + t), s_cnt++ & 1u, kErrWaitSFull));
        if (!ok) break;
        tc_fence_after();
        float s[128];
        if constexpr (BIAS) {
          // s <- s * scale + M, in natural-log units; the exponent below turns
          // them into log2 units (sl2_eff = log2(e)).  S comes out of tensor
          // memory a quarter at a time, so each quarter's M registers die as
          // it lands.
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t sr[32];
            tmem_ld_x32_wait(s_addr + static_cast<uint32_t>(32 * q4), sr);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint32_t wv[4] = {mb[4 * q4 + v].x, mb[4 * q4 + v].y, mb[4 * q4 + v].z, mb[4 * q4 + v].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int c = 32 * q4 + 8 * v + 2 * i;
                s[c] = fmaf(__uint_as_float(sr[c - 32 * q4]), p.scale, __uint_as_float(wv[i] << 16));
                s[c + 1] = fmaf(__uint_as_float(sr[c + 1 - 32 * q4]), p.scale, __uint_as_float(wv[i] & 0xffff0000u));
              }
            }
          }
        } else {
          uint32_t sr[128];
          tmem_ld_x128_wait(s_addr, sr);
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
        }
        // Tiles crossing the causal diagonal, a window's left edge or N get a
        // per-element mask (a select, so NaN-free -inf).
        if ((CAUSAL && kv0 + 127 > row0) || kv0 + 128 > n_kv ||
            (WINDOW && kv0 < min(row0 + 127, n_kv - 1) - p.window_left)) {
          // Visible keys of this row: [first, last], as offsets into the tile.
          const int last = (CAUSAL ? min(grow, n_kv - 1) : n_kv - 1) - kv0;
          if constexpr (WINDOW) {
            const int first = grow - p.window_left - kv0;
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > last || c < first) s[c] = -INFINITY;
          } else {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > last) s[c] = -INFINITY;
          }
        }
        // Row max: four chains of three-input maxima over s[4..123], then
        // s[124..127] one per chain.
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c + 8 <= 124; c += 8) {
          mx0 = max3(mx0, s[c], s[c + 1]);
          mx1 = max3(mx1, s[c + 2], s[c + 3]);
          mx2 = max3(mx2, s[c + 4], s[c + 5]);
          mx3 = max3(mx3, s[c + 6], s[c + 7]);
        }
        mx0 = fmaxf(mx0, s[124]);
        mx1 = fmaxf(mx1, s[125]);
        mx2 = fmaxf(mx2, s[126]);
        mx3 = fmaxf(mx3, s[127]);
        float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float sl2_eff = BIAS ? 1.4426950408889634f : sl2;  // additive M: scores in natural-log units
        m_tile *= sl2_eff;
        const float m_new = fmaxf(m_used, m_tile);
        const bool upd = m_new > m_used + (FP8 ? kRescaleThresholdFp8 : kRescaleThreshold);
        const float alpha = upd ? ex2_approx(m_used - m_new) : 1.f;  // 0 on the first tile
        if (upd) m_used = m_new;
        l_sum *= alpha;
        // FP8: P = 2^8 * 2^(s - m), the 2^8 folded into the offset.
        const float neg_m = (m_used == -INFINITY) ? 0.f : (FP8 ? kFp8PLog2 - m_used : -m_used);
        const uint64_t sl2x2 = f2_pack(sl2_eff, sl2_eff);
        const uint64_t negm2 = f2_pack(neg_m, neg_m);
        // P in two halves, columns [0, 64) then [64, 128); each half goes to
        // tensor memory as soon as it is packed (fewer live registers).
        uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if constexpr (FP8) {
            // Four e4m3 weights per 32-bit column: 16 columns per half.
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c = half * 64 + 4 * i;
              float x0, x1, x2, x3;
              f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, negm2), x0, x1);
              f2_unpack(f2_fma(f2_pack(s[c + 2], s[c + 3]), sl2x2, negm2), x2, x3);
              float p0, p1, p2, p3;
              if (kExp2EmuPeriodFp8 > 0 &&
                  i % (kExp2EmuPeriodFp8 > 0 ? kExp2EmuPeriodFp8 : 1) == kExp2EmuPeriodFp8 - 1) {
                p0 = exp2_poly(x0);
                p1 = exp2_poly(x1);
                p2 = exp2_poly(x2);
                p3 = exp2_poly(x3);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
                p2 = ex2_approx(x2);
                p3 = ex2_approx(x3);
              }
              acc[0] = f2_add(acc[0], f2_pack(p0, p1));
              acc[1] = f2_add(acc[1], f2_pack(p2, p3));
              pk[i] = pack_e4m3x4(p0, p1, p2, p3);
            }
            tmem_st_x16(s_addr + static_cast<uint32_t>(half * 16), pk);
          } else {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = half * 64 + 2 * i;
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, negm2), x0, x1);
              float p0, p1;
              if (kExp2EmuPeriod > 0 && i % (kExp2EmuPeriod > 0 ? kExp2EmuPeriod : 1) == kExp2EmuPeriod - 1) {
                p0 = exp2_poly(x0);
                p1 = exp2_poly(x1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              acc[i & 1] = f2_add(acc[i & 1], f2_pack(p0, p1));
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st_x32(s_addr + static_cast<uint32_t>(half * 32), pk);
          }
          if (half == 0 && jj > 0 && __any_sync(0xffffffffu, upd)) {
            // O_t is idle here (its last update was issued before S_t of this
            // tile, and this tile's update waits for the barrier below).
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t o[32];
              tmem_ld_x32_wait(o_addr + c, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st_x32(o_addr + c, o);
            }
          }
          if (half == 1) {
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(L::kBarPFull + t));
          }
        }
        float ls0, ls1, ls2, ls3;
        f2_unpack(acc[0], ls0, ls1);
        f2_unpack(acc[1], ls2, ls3);
        l_sum += (ls0 + ls1) + (ls2 + ls3);
      }
      if (!ok) break;
      // Hand m and l of this row to the epilogue (2-slot ring per tile).
      const uint32_t slot = st_cnt & 1u;
      if (st_cnt >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarStatsEmpty + 2 * t + slot),
                                               ((st_cnt >> 1) - 1u) & 1u, kErrWaitSFull));
        if (!ok) break;
      }
      float* sp = stats + ((t * 2 + slot) * 2) * 128;
      sp[row] = m_used;
      sp[128 + row] = l_sum;
      mbar_arrive(bar(L::kBarStatsFull + 2 * t + slot));
      ++st_cnt;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace attn
