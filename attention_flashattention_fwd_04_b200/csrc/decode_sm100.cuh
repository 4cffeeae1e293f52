// Paged-KV decode attention for sm_100a: a split-KV pass and an LSE-weighted
// merge.
//
// The KV cache is a pool of fixed-size pages and each sequence reaches its
// pages through a block table; logical token t of sequence s lives in page
// block_table[s][t / page_size], slot t % page_size ("Fast Attention Kernels
// and Operator Fusion", section "Paged Attention Kernels": the kernel cannot
// assume K_{t+1} follows K_t and must translate every logical position
// through the table).  Decode reads the whole cache once per query token, so
// the pass is bound by HBM reads of K and V.
//
// Split pass: CTA (split, seq, kv-head group) walks its 16-token chunks of the
// sequence.  A producer warp issues TMA tile loads of each chunk's K and V
// rows for HB kv heads into a 3-stage shared-memory ring; consumer warp w
// handles kv head w and its Hq/Hkv query heads with mma.sync m16n8k16 (the
// query group, at most 16 rows, is far below the 64/128-row tcgen05 shapes,
// and the arithmetic here is a few FLOP per byte).  The online softmax keeps a
// running max and sum per query head; the split writes its normalised partial
// O_t (fp32) and lse_t.
//
// Merge: lse = log sum_t exp(lse_t) and O = sum_t exp(lse_t - lse) O_t, the
// same rescaling identity that lets the softmax be computed in pieces.
#pragma once

#include "ptx.cuh"

namespace attn {

constexpr int kDecodeChunk = 16;   // tokens per pipeline stage (the mma K extent)
constexpr int kDecodeStages = 3;

struct DecodeParams {
  const __nv_bfloat16* q;      // [S, Hq, D]
  const int32_t* block_table;  // [S, max_pages]
  const int32_t* seq_lens;     // [S]
  float* part_o;               // [S, Hq, max_splits, D]
  float* part_lse;             // [S, Hq, max_splits]
  int S, Hq, Hkv, group, page_size, max_pages, num_pages, max_splits, split_tokens;
  float scale_log2;
};

template <int D, int HB>
struct DecodeLayout {
  static constexpr int kBoxBytes = HB * kDecodeChunk * 128;  // one 64-column half, HB heads
  static constexpr int kHalves = D / 64;
  static constexpr int kPoolBytes = kHalves * kBoxBytes;      // one pool, one chunk
  static constexpr int kStageBytes = 2 * kPoolBytes;          // K then V
  static constexpr int kBar = kDecodeStages * kStageBytes;
  static constexpr int kNumBars = 2 * kDecodeStages;
  static constexpr int kTable = kBar + kNumBars * 8;          // block-table entries of the split
  static constexpr int kMaxTableEntries = 256;
  static constexpr int kBytes = kTable + kMaxTableEntries * 4;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

// D = A * B + D for one m16n8k16 bf16 tile with fp32 accumulation.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Address of the 16-byte chunk `c8` (8 bf16 columns, 0..D/8-1) of token row
// `t` of kv head `hl` inside one pool's part of a stage.  TMA wrote the
// [HB heads][16 tokens][64 columns] boxes with the 128-byte swizzle: the
// 16-byte chunk index inside each 128-byte row is XORed with row % 8.
template <int HB>
__device__ __forceinline__ uint32_t decode_smem_addr(uint32_t pool_base, int hl, int t, int c8) {
  const int row = hl * kDecodeChunk + t;
  const int half = c8 >> 3;
  const int chunk = (c8 & 7) ^ (row & 7);
  return pool_base + static_cast<uint32_t>(half * (HB * kDecodeChunk * 128) + row * 128 + chunk * 16);
}

template <int D, int HB>
__global__ void __launch_bounds__(32 * (HB + 1), 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using L = DecodeLayout<D, HB>;
  // The merge grid (launched as a programmatic dependent) may start once every
  // CTA of this grid has started: it then waits for this grid's completion in
  // griddepcontrol.wait, so its launch overlaps this grid's last wave.  All
  // split CTAs are resident or done by then, so none waits for an SM.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int split = blockIdx.x;
  const int s = blockIdx.y;
  const int head0 = blockIdx.z * HB;  // first kv head of this CTA
  const int seq_len = p.seq_lens[s];
  const int tok_begin = split * p.split_tokens;
  if (seq_len <= 0 || seq_len > p.max_pages * p.page_size) {
    if (split == 0 && blockIdx.z == 0 && threadIdx.x == 0) atomicOr(&g_attn_device_error, kErrDecodeTable);
    return;
  }
  if (tok_begin >= seq_len) return;  // nothing of this sequence falls in this split
  const int tok_end = min(seq_len, tok_begin + p.split_tokens);
  const int n_chunks = (tok_end - tok_begin + kDecodeChunk - 1) / kDecodeChunk;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto full_bar = [&](int st) -> uint32_t { return base + L::kBar + 8u * st; };
  auto empty_bar = [&](int st) -> uint32_t { return base + L::kBar + 8u * (kDecodeStages + st); };
  int32_t* table_s = reinterpret_cast<int32_t*>(smem + L::kTable);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Block-table entries covering this split, read once and range-checked.
  {
    const int page_first = tok_begin / p.page_size;
    const int page_last = (tok_end - 1) / p.page_size;
    for (int i = threadIdx.x; i <= page_last - page_first; i += blockDim.x) {
      int e = p.block_table[static_cast<size_t>(s) * p.max_pages + page_first + i];
      if (e < 0 || e >= p.num_pages) {
        atomicOr(&g_attn_device_error, kErrDecodeTable);
        e = 0;  // keep every copy inside the pool; the result is flagged invalid
      }
      table_s[i] = e;
    }
  }
  if (threadIdx.x == 0) {
    for (int st = 0; st < kDecodeStages; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), HB);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == HB) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int page_first = tok_begin / p.page_size;
      bool ok = true;
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kDecodeStages;
        const uint32_t round = static_cast<uint32_t>(c / kDecodeStages);
        if (round > 0) ok = mbar_wait(empty_bar(st), (round - 1) & 1u, kErrDecodeWait);
        if (!ok) break;
        const int tok = tok_begin + c * kDecodeChunk;
        const int page = tok / p.page_size;
        const int slot = tok - page * p.page_size;
        const int row = table_s[page - page_first] * p.page_size + slot;
        const uint32_t dst = base + static_cast<uint32_t>(st * L::kStageBytes);
        mbar_arrive_expect_tx(full_bar(st), L::kStageBytes);
#pragma unroll
        for (int hf = 0; hf < L::kHalves; ++hf) {
          tma_load_3d(dst + hf * L::kBoxBytes, &tm_k, full_bar(st), hf * 64, row, head0);
          tma_load_3d(dst + L::kPoolBytes + hf * L::kBoxBytes, &tm_v, full_bar(st), hf * 64, row, head0);
        }
        ++issued;
      }
      for (int c = max(0, issued - kDecodeStages); c < issued; ++c)
        mbar_wait(full_bar(c % kDecodeStages), static_cast<uint32_t>(c / kDecodeStages) & 1u,
                  kErrDecodeWait);
    }
    __syncwarp();
    return;
  }

  // -------------------------------------------------------------- consumers
  const int hl = warp;              // local kv head
  const int hk = head0 + hl;        // kv head
  const int g = p.group;            // query heads per kv head (<= 16)
  const int grp = lane >> 2;        // mma groupID: query-head row (and +8)
  const int tig = lane & 3;         // thread in group
  const float sl2 = p.scale_log2;

  // Q fragments (A operand, rows = the group's query heads, zero past g).
  uint32_t qa[D / 16][4];
  {
    const __nv_bfloat16* qbase = p.q + (static_cast<size_t>(s) * p.Hq + static_cast<size_t>(hk) * g) * D;
    const int r0 = grp, r1 = grp + 8;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c0 = kk * 16 + tig * 2;
      qa[kk][0] = r0 < g ? *reinterpret_cast<const uint32_t*>(qbase + r0 * D + c0) : 0u;
      qa[kk][1] = r1 < g ? *reinterpret_cast<const uint32_t*>(qbase + r1 * D + c0) : 0u;
      qa[kk][2] = r0 < g ? *reinterpret_cast<const uint32_t*>(qbase + r0 * D + c0 + 8) : 0u;
      qa[kk][3] = r1 < g ? *reinterpret_cast<const uint32_t*>(qbase + r1 * D + c0 + 8) : 0u;
    }
  }

  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max (scaled log2) of rows grp, grp+8
  float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums
  bool ok = true;

  for (int c = 0; c < n_chunks; ++c) {
    const int st = c % kDecodeStages;
    ok = mbar_wait(full_bar(st), static_cast<uint32_t>(c / kDecodeStages) & 1u, kErrDecodeWait);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const uint32_t kbase = base + static_cast<uint32_t>(st * L::kStageBytes);
    const uint32_t vbase = kbase + L::kPoolBytes;
    const int valid = min(kDecodeChunk, tok_end - (tok_begin + c * kDecodeChunk));

    if (valid < kDecodeChunk) {
      // Slots past the end of the sequence may hold anything (even NaN); zero
      // this head's V rows there so P = 0 really contributes nothing.
      for (int idx = lane; idx < (kDecodeChunk - valid) * 8 * L::kHalves; idx += 32) {
        const int t = valid + idx / (8 * L::kHalves);
        const int c8 = idx % (8 * L::kHalves);
        *reinterpret_cast<uint4*>(smem + (decode_smem_addr<HB>(vbase, hl, t, c8) - base)) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }

    // S = Q K^T for 16 tokens: two n8 tiles (tokens 0-7, 8-15).
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int mi = lane >> 3, ri = lane & 7;  // matrix / row this lane addresses
      const int t = (mi >> 1) * 8 + ri;
      const int c8 = kk * 2 + (mi & 1);
      uint32_t b00, b01, b10, b11;
      ldmatrix_x4(decode_smem_addr<HB>(kbase, hl, t, c8), b00, b01, b10, b11);
      mma_16816(sc[0], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b00, b01);
      mma_16816(sc[1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b10, b11);
    }
    // Mask tokens past the end of the sequence (select, so NaN scores vanish).
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = n * 8 + tig * 2 + (e & 1);
        sc[n][e] = (t < valid) ? sc[n][e] * sl2 : -INFINITY;
      }
    }
    float cm0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    float cm1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 1));
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 2));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 1));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 2));
    const float mn0 = fmaxf(m0, cm0), mn1 = fmaxf(m1, cm1);  // finite: chunk has >= 1 valid token
    const float a0 = ex2_approx(m0 - mn0), a1 = ex2_approx(m1 - mn1);  // 0 on the first chunk
    m0 = mn0;
    m1 = mn1;
    float pr[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      pr[n][0] = ex2_approx(sc[n][0] - mn0);
      pr[n][1] = ex2_approx(sc[n][1] - mn0);
      pr[n][2] = ex2_approx(sc[n][2] - mn1);
      pr[n][3] = ex2_approx(sc[n][3] - mn1);
    }
    l0 = l0 * a0 + (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
    l1 = l1 * a1 + (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc[n][0] *= a0;
      acc[n][1] *= a0;
      acc[n][2] *= a1;
      acc[n][3] *= a1;
    }
    // P as the A operand (rows = query heads, k = the 16 tokens).
    const uint32_t pa0 = pack_bf16x2(pr[0][0], pr[0][1]);
    const uint32_t pa1 = pack_bf16x2(pr[0][2], pr[0][3]);
    const uint32_t pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
    const uint32_t pa3 = pack_bf16x2(pr[1][2], pr[1][3]);
    // O += P V: V^T fragments via transposed ldmatrix, two n8 tiles per load.
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      const int mi = lane >> 3, ri = lane & 7;
      const int t = (mi & 1) * 8 + ri;
      const int c8 = np * 2 + (mi >> 1);
      uint32_t v0, v1, v2, v3;
      ldmatrix_x4_trans(decode_smem_addr<HB>(vbase, hl, t, c8), v0, v1, v2, v3);
      mma_16816(acc[2 * np], pa0, pa1, pa2, pa3, v0, v1);
      mma_16816(acc[2 * np + 1], pa0, pa1, pa2, pa3, v2, v3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(st));
  }
  if (!ok) return;

  // Full row sums across the quad, then write the normalised partials.
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int r0 = grp, r1 = grp + 8;
  const size_t row_stride = static_cast<size_t>(p.max_splits) * D;
  const size_t head_base = (static_cast<size_t>(s) * p.Hq + static_cast<size_t>(hk) * g);
  if (r0 < g) {
    float* dst = p.part_o + (head_base + r0) * row_stride + static_cast<size_t>(split) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<float2*>(dst + n * 8 + tig * 2) = make_float2(acc[n][0] * inv0, acc[n][1] * inv0);
    if (tig == 0) p.part_lse[(head_base + r0) * p.max_splits + split] = (m0 + log2f(l0)) * 0.69314718055994530942f;
  }
  if (r1 < g) {
    float* dst = p.part_o + (head_base + r1) * row_stride + static_cast<size_t>(split) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<float2*>(dst + n * 8 + tig * 2) = make_float2(acc[n][2] * inv1, acc[n][3] * inv1);
    if (tig == 0) p.part_lse[(head_base + r1) * p.max_splits + split] = (m1 + log2f(l1)) * 0.69314718055994530942f;
  }
}

// One warp per (sequence, query head): combine the splits that hold tokens.
// Lane i computes the weight of split i of each group of 32.  Up to 32
// splits, every partial row is requested together with the partial LSEs (the
// rows do not depend on the weights), so the merge costs two dependent trips
// to memory (the length, then everything); longer sequences read the rows 16
// splits per round after the weights.
constexpr int kMergeThreads = 128;
template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    decode_merge_kernel(const DecodeParams p, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  // Launched as a programmatic dependent of the split pass: wait until that
  // grid has completed and its partials are visible (returns at once when
  // launched without the attribute).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= p.S * p.Hq) return;
  const int s = wid / p.Hq;
  const int seq_len = p.seq_lens[s];
  constexpr int kPer = D / 32;  // output columns per lane
  __nv_bfloat16* orow = o + static_cast<size_t>(wid) * D;
  if (seq_len <= 0 || seq_len > p.max_pages * p.page_size) {
    // Invalid length (flagged by the split pass): defined zeros, LSE = -inf.
    for (int i = 0; i < kPer; ++i) orow[lane * kPer + i] = __float2bfloat16_rn(0.f);
    if (lane == 0) lse[wid] = -INFINITY;
    return;
  }
  const int n_splits = (seq_len + p.split_tokens - 1) / p.split_tokens;
  const float* plse = p.part_lse + static_cast<size_t>(wid) * p.max_splits;
  const float* po = p.part_o + static_cast<size_t>(wid) * p.max_splits * D + lane * kPer;
  constexpr float kLog2e = 1.4426950408889634f;
  if (n_splits <= 32) {
    const float pl = lane < n_splits ? plse[lane] : -INFINITY;
    float v[32][kPer];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      if (u < n_splits) {
        const float* src = po + static_cast<size_t>(u) * D;
        if constexpr (kPer == 4) {
          const float4 x = *reinterpret_cast<const float4*>(src);
          v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(src);
          v[u][0] = x.x; v[u][1] = x.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < kPer; ++e) v[u][e] = 0.f;
      }
    }
    float mx = pl;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float my_w = lane < n_splits ? ex2_approx((pl - mx) * kLog2e) : 0.f;
    float wsum = my_w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    float out[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) out[e] = 0.f;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float w = __shfl_sync(0xffffffffu, my_w, u);
#pragma unroll
      for (int e = 0; e < kPer; ++e) out[e] = fmaf(w, v[u][e], out[e]);
    }
    const float inv = 1.f / wsum;
#pragma unroll
    for (int e = 0; e < kPer; e += 2)
      *reinterpret_cast<uint32_t*>(orow + lane * kPer + e) = pack_bf16x2(out[e] * inv, out[e + 1] * inv);
    if (lane == 0) lse[wid] = mx + logf(wsum);
    return;
  }
  // The first 32 splits' LSEs stay in registers (lane t: split t) for the
  // weights; the partial rows are then read 16 splits per round, so a
  // sequence of up to 32 splits costs three dependent trips to memory.
  const float pl0 = lane < n_splits ? plse[lane] : -INFINITY;
  float mx = pl0;
  for (int t = lane + 32; t < n_splits; t += 32) mx = fmaxf(mx, plse[t]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float wsum = 0.f;
  float out[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) out[e] = 0.f;
  constexpr int kRound = 16;  // splits whose rows are in flight at once
  for (int t0 = 0; t0 < n_splits; t0 += 32) {
    const int cnt = min(32, n_splits - t0);
    const float pl = t0 == 0 ? pl0 : (lane < cnt ? plse[t0 + lane] : -INFINITY);
    const float my_w = lane < cnt ? ex2_approx((pl - mx) * kLog2e) : 0.f;
    wsum += my_w;
    for (int i = 0; i < cnt; i += kRound) {
      float v[kRound][kPer];
      float w[kRound];
#pragma unroll
      for (int u = 0; u < kRound; ++u) {
        w[u] = __shfl_sync(0xffffffffu, my_w, (i + u) & 31);
        if (i + u < cnt) {
          const float* src = po + static_cast<size_t>(t0 + i + u) * D;
          if constexpr (kPer == 4) {
            const float4 x = *reinterpret_cast<const float4*>(src);
            v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
          } else {
            const float2 x = *reinterpret_cast<const float2*>(src);
            v[u][0] = x.x; v[u][1] = x.y;
          }
        } else {
          w[u] = 0.f;
#pragma unroll
          for (int e = 0; e < kPer; ++e) v[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kRound; ++u)
#pragma unroll
        for (int e = 0; e < kPer; ++e) out[e] = fmaf(w[u], v[u][e], out[e]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  const float inv = 1.f / wsum;
#pragma unroll
  for (int e = 0; e < kPer; e += 2)
    *reinterpret_cast<uint32_t*>(orow + lane * kPer + e) = pack_bf16x2(out[e] * inv, out[e + 1] * inv);
  if (lane == 0) lse[wid] = mx + logf(wsum);
}

}  // namespace attn
