// Appending new tokens' K and V to a paged KV cache (sm_100a).
//
// "Fast Attention Kernels and Operator Fusion" lists updating the KV cache
// while keys and values are produced among the fusions of a decoder layer
// (section "Operator Fusion"), and its paged cache is a pool of fixed-size
// blocks found through a per-sequence block table, allocated as the sequence
// grows (section "Paged Attention Kernels").  Here the new keys and values of
// a step arrive packed by sequence; new token i of sequence s is logical
// token ctx + i (ctx = seq_lens[s] - q_len), written to physical page
// block_table[s][(ctx + i) / page_size], slot (ctx + i) % page_size.
//
// Each warp copies a run of consecutive new tokens: one binary search finds
// the sequence of the first, the rest walk forward.  A token's [Hkv, D] rows
// of K and of V are contiguous both in the packed input and in the page
// slot, so each is one straight copy of Hkv * D * 2 bytes in 16-byte
// vectors; all of a token's vectors are loaded before any is stored, so the
// loads overlap.  HBM-bound.
#pragma once

#include "ptx.cuh"

namespace attn {

struct AppendParams {
  const __nv_bfloat16* k_new;  // [total_q, Hkv, D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool;       // [num_pages, page_size, Hkv, D]
  __nv_bfloat16* v_pool;
  const int32_t* cu_q;         // [num_seqs + 1]
  const int32_t* seq_lens;     // [num_seqs], after the append
  const int32_t* block_table;  // [num_seqs, max_pages]
  int num_seqs, total_q, Hkv, D, max_pages, num_pages, page_size;
};

constexpr int kAppendThreads = 256;
constexpr int kAppendTokensPerWarp = 4;
constexpr int kAppendVecsPerLane = 4;  // 16-byte vectors per lane and tensor in one batch

__global__ void __launch_bounds__(kAppendThreads) paged_append_kernel(const AppendParams p) {
  const int lane = threadIdx.x & 31;
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int t_begin = gw * kAppendTokensPerWarp;
  if (t_begin >= p.total_q) return;
  const int t_end = min(p.total_q, t_begin + kAppendTokensPerWarp);
  const int vecs = p.Hkv * p.D / 8;  // 16-byte vectors per token and tensor
  // Sequence of the first token: the last s with cu_q[s] <= t_begin.
  int lo = 0, hi = p.num_seqs;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.cu_q[mid] <= t_begin) lo = mid; else hi = mid;
  }
  int s = lo;
  int q0 = p.cu_q[s], q1 = p.cu_q[s + 1], len = p.seq_lens[s];
  for (int t = t_begin; t < t_end; ++t) {
    while (t >= q1 && s + 1 < p.num_seqs) {  // next non-empty sequence
      ++s;
      q0 = q1;
      q1 = p.cu_q[s + 1];
      len = p.seq_lens[s];
    }
    const int nq = q1 - q0;
    const int i = t - q0;
    if (i < 0 || i >= nq || nq > len || len > p.max_pages * p.page_size) {
      if (lane == 0) atomicOr(&g_attn_device_error, kErrPagedTable);
      continue;
    }
    const int pos = len - nq + i;
    const int pg = p.block_table[static_cast<size_t>(s) * p.max_pages + pos / p.page_size];
    if (pg < 0 || pg >= p.num_pages) {
      if (lane == 0) atomicOr(&g_attn_device_error, kErrPagedTable);
      continue;  // nothing is written outside the pool
    }
    const size_t dst = (static_cast<size_t>(pg) * p.page_size + pos % p.page_size) * vecs;
    const size_t src = static_cast<size_t>(t) * vecs;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k_new) + src;
    const uint4* vs = reinterpret_cast<const uint4*>(p.v_new) + src;
    uint4* kd = reinterpret_cast<uint4*>(p.k_pool) + dst;
    uint4* vd = reinterpret_cast<uint4*>(p.v_pool) + dst;
    for (int base = 0; base < vecs; base += 32 * kAppendVecsPerLane) {
      uint4 a[kAppendVecsPerLane], b[kAppendVecsPerLane];
#pragma unroll
      for (int u = 0; u < kAppendVecsPerLane; ++u) {
        const int x = base + u * 32 + lane;
        if (x < vecs) {
          a[u] = ks[x];
          b[u] = vs[x];
        }
      }
#pragma unroll
      for (int u = 0; u < kAppendVecsPerLane; ++u) {
        const int x = base + u * 32 + lane;
        if (x < vecs) {
          kd[x] = a[u];
          vd[x] = b[u];
        }
      }
    }
  }
}

}  // namespace attn
