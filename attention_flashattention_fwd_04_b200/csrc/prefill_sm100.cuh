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
// One CTA owns one 128-row query tile of one (batch, query head):
//   warp 0      TMA producer: Q once, then K_j / V_j tiles into a 2-stage ring
//   warp 1      allocates tensor memory; lane 0 issues every tcgen05.mma
//   warps 4-7   softmax: thread t owns query row t (= TMEM lane t)
// Tensor memory (512 columns): S_0 | S_1 (128 fp32 columns each, double
// buffered so S_{j+1} = Q K_{j+1}^T runs while the softmax of tile j runs),
// O (D fp32 columns).  P_j (bf16) is written back over the first 64 columns
// of its own S buffer and read from there as the A operand of O += P_j V_j.
// The O rescale is lazy: the running max used for P only moves when the tile
// max exceeds it by more than 2^8; the final O / l uses that same max, so the
// result is exact.
#pragma once

#include "ptx.cuh"
#include "tmem_ldst.cuh"

namespace attn {

struct PrefillParams {
  __nv_bfloat16* o;  // [B, Hq, N, D]
  float* lse;        // [B, Hq, N]
  int B, Hq, Hkv, N;
  int group;         // Hq / Hkv
  int num_q_tiles;   // ceil(N / 128)
  float scale_log2;  // scale * log2(e)
};

constexpr int kPrefillThreads = 256;
constexpr float kRescaleThreshold = 8.0f;  // in log2 units
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, int NS>
struct PrefillLayout {
  static constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128B-swizzled box)
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + NS * kTileBytes;
  static constexpr int kBar = kV + NS * kTileBytes;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + NS;
  static constexpr int kBarVFull = kBarKEmpty + NS;
  static constexpr int kBarVEmpty = kBarVFull + NS;
  static constexpr int kBarSFull = kBarVEmpty + NS;  // two
  static constexpr int kBarPFull = kBarSFull + 2;    // two
  static constexpr int kBarODone = kBarPFull + 2;
  static constexpr int kBarMmaDone = kBarODone + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kBytes = kTmemSlot + 16;
  // 1024 B of slack for rounding the base up; at least 116 KB so that a second
  // CTA never shares the SM (each CTA takes all 512 tensor-memory columns).
  static constexpr int kAlloc = (kBytes + 1024) > 116 * 1024 ? (kBytes + 1024) : 116 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
};

template <int D, bool CAUSAL, int NS>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  using L = PrefillLayout<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) -> uint32_t { return base + L::kBar + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh_count = p.B * p.Hq;
  const int tile_rank = static_cast<int>(blockIdx.x) / bh_count;
  // Causal: the longest query tiles go first so the short ones fill the tail.
  const int qt = CAUSAL ? (p.num_q_tiles - 1 - tile_rank) : tile_rank;
  const int bh = static_cast<int>(blockIdx.x) % bh_count;
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int hk = h / p.group;  // GQA: consecutive query heads share a KV head
  const int n_kv_all = (p.N + 127) / 128;
  const int n_kv = CAUSAL ? min(qt + 1, n_kv_all) : n_kv_all;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQ), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    mbar_init(bar(L::kBarSFull + 0), 1);
    mbar_init(bar(L::kBarSFull + 1), 1);
    mbar_init(bar(L::kBarPFull + 0), 128);
    mbar_init(bar(L::kBarPFull + 1), 128);
    mbar_init(bar(L::kBarODone), 1);
    mbar_init(bar(L::kBarMmaDone), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(base + L::kTmemSlot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int qz = b * p.Hq + h;
      const int kz = b * p.Hkv + hk;
      mbar_arrive_expect_tx(bar(L::kBarQ), L::kTileBytes);
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(base + L::kQ + c * L::kBoxBytes, &tm_q, bar(L::kBarQ), c * 64, qt * 128, qz);
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % NS;
        const uint32_t round = static_cast<uint32_t>(j / NS);
        if (round > 0) ok = mbar_wait(bar(L::kBarKEmpty + st), (round - 1) & 1u, kErrWaitKEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::kBarKFull + st), L::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(base + L::kK + st * L::kTileBytes + c * L::kBoxBytes, &tm_k,
                      bar(L::kBarKFull + st), c * 64, j * 128, kz);
        ++k_issued;
        if (round > 0) ok = mbar_wait(bar(L::kBarVEmpty + st), (round - 1) & 1u, kErrWaitVEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(L::kBarVFull + st), L::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(base + L::kV + st * L::kTileBytes + c * L::kBoxBytes, &tm_v,
                      bar(L::kBarVFull + st), c * 64, j * 128, kz);
        ++v_issued;
      }
      // Every copy this thread started must land before the CTA may exit.
      mbar_wait(bar(L::kBarQ), 0, kErrWaitDrain);
      for (int j = max(0, k_issued - NS); j < k_issued; ++j)
        mbar_wait(bar(L::kBarKFull + j % NS), static_cast<uint32_t>(j / NS) & 1u, kErrWaitDrain);
      for (int j = max(0, v_issued - NS); j < v_issued; ++j)
        mbar_wait(bar(L::kBarVFull + j % NS), static_cast<uint32_t>(j / NS) & 1u, kErrWaitDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D, false, true);
      const uint32_t q_addr = base + L::kQ;
      bool ok = mbar_wait(bar(L::kBarQ), 0, kErrWaitQ);
      auto issue_s = [&](int j) -> bool {
        const int st = j % NS;
        if (!mbar_wait(bar(L::kBarKFull + st), static_cast<uint32_t>(j / NS) & 1u, kErrWaitKFull))
          return false;
        tc_fence_after();
        const uint32_t k_addr = base + L::kK + st * L::kTileBytes;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(j & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * L::kBoxBytes + (kk & 3) * 32);
          mma_bf16_ss(d_tmem, make_sdesc_sw128(q_addr + off, 16, 1024),
                      make_sdesc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::kBarSFull + (j & 1)));
        mma_commit(bar(L::kBarKEmpty + st));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv) {
          ok = issue_s(j + 1);
          if (!ok) break;
        }
        const int st = j % NS;
        ok = mbar_wait(bar(L::kBarPFull + (j & 1)), static_cast<uint32_t>(j >> 1) & 1u, kErrWaitPFull);
        if (!ok) break;
        ok = mbar_wait(bar(L::kBarVFull + st), static_cast<uint32_t>(j / NS) & 1u, kErrWaitVFull);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_addr = base + L::kV + st * L::kTileBytes;
        const uint32_t p_tmem = tmem + static_cast<uint32_t>(j & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_bf16_ts(tmem + L::kColO, p_tmem + kk * 8,
                      make_sdesc_sw128(v_addr + kk * 2048, L::kBoxBytes, 1024), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(L::kBarODone));
        mma_commit(bar(L::kBarVEmpty + st));
      }
      // All issued MMAs must finish before tensor memory is released.
      mma_commit(bar(L::kBarMmaDone));
      mbar_wait(bar(L::kBarMmaDone), 0, kErrWaitMmaDone);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int grow = qt * 128 + row;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;  // running max in scaled log2 units
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int buf = j & 1;
      ok = mbar_wait(bar(L::kBarSFull + buf), static_cast<uint32_t>(j >> 1) & 1u, kErrWaitSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128_wait(lane_addr + static_cast<uint32_t>(buf) * 128u, sr);
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      const int kv0 = j * 128;
      if ((CAUSAL && j == qt) || kv0 + 128 > p.N) {
        const int last = CAUSAL ? min(grow, p.N - 1) : p.N - 1;  // last visible key
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kv0 + c > last) s[c] = -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, s[c]);
        mx1 = fmaxf(mx1, s[c + 1]);
        mx2 = fmaxf(mx2, s[c + 2]);
        mx3 = fmaxf(mx3, s[c + 3]);
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      const float m_new = fmaxf(m_used, m_tile);
      const bool upd = m_new > m_used + kRescaleThreshold;
      const float alpha = upd ? ex2_approx(m_used - m_new) : 1.f;  // 0 on the first tile
      if (upd) m_used = m_new;
      l_sum *= alpha;
      const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
      uint32_t pk_lo[32], pk_hi[32];
      float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        const float p0 = ex2_approx(fmaf(s[c], sl2, neg_m));
        const float p1 = ex2_approx(fmaf(s[c + 1], sl2, neg_m));
        const float p2 = ex2_approx(fmaf(s[c + 2], sl2, neg_m));
        const float p3 = ex2_approx(fmaf(s[c + 3], sl2, neg_m));
        ls0 += p0;
        ls1 += p1;
        ls2 += p2;
        ls3 += p3;
        if (c < 64) {
          pk_lo[c / 2] = pack_bf16x2(p0, p1);
          pk_lo[c / 2 + 1] = pack_bf16x2(p2, p3);
        } else {
          pk_hi[(c - 64) / 2] = pack_bf16x2(p0, p1);
          pk_hi[(c - 64) / 2 + 1] = pack_bf16x2(p2, p3);
        }
      }
      l_sum += (ls0 + ls1) + (ls2 + ls3);
      const uint32_t p_addr = lane_addr + static_cast<uint32_t>(buf) * 128u;
      tmem_st_x32(p_addr, pk_lo);
      tmem_st_x32(p_addr + 32u, pk_hi);
      if (j > 0) {
        // O may only be touched once O += P_{j-1} V_{j-1} has completed.
        ok = mbar_wait(bar(L::kBarODone), static_cast<uint32_t>(j - 1) & 1u, kErrWaitODone);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (__any_sync(0xffffffffu, upd)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld_x32_wait(lane_addr + L::kColO + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_x32(lane_addr + L::kColO + c, o);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarPFull + buf));
    }
    if (ok) {
      ok = mbar_wait(bar(L::kBarODone), static_cast<uint32_t>(n_kv - 1) & 1u, kErrWaitODone);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_sum;
      const size_t row_index = static_cast<size_t>(b * p.Hq + h) * p.N + grow;
      __nv_bfloat16* orow = p.o + row_index * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld_x32_wait(lane_addr + L::kColO + c, o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (grow < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
          dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
        }
      }
      if (grow < p.N) p.lse[row_index] = (m_used + log2f(l_sum)) * kLn2;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace attn
