// Host side of the C ABI declared in include/attn_b200.h: argument checks,
// TMA tensor-map encoding, split planning and kernel launches.  Nothing here
// allocates device memory or synchronises (except attn_device_status, whose
// job is to synchronise).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <new>

#include "attn_b200.h"
#include "decode_sm100.cuh"
#include "paged_append.cuh"
#include "prefill_sm100.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

int fail_cuda(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return ATTN_ERR_LAUNCH;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres{};
    const cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                                           cudaEnableDefault, &qres);
    if (e == cudaSuccess && qres == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 tensor map, 128-byte swizzle, zero fill outside the tensor.
// dims[0] is the contiguous dimension; strides are the byte strides of
// dims[1] and dims[2].
bool encode_3d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1, stride2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, dtype, 3, const_cast<void*>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute is per device), so launches do not repeat the driver call.
template <auto Kernel>
cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<uint64_t> done{0};  // one bit per device ordinal < 64
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

constexpr float kLog2e = 1.4426950408889634f;

int sm_count() {
  static int counts[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    counts[dev] = n;
  }
  return counts[dev];
}

template <int D, bool CAUSAL, bool WINDOW, bool PAGED = false, bool FP8 = false, bool SPARSE = false,
          bool BIAS = false>
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const attn::PrefillParams& p, cudaStream_t stream) {
  using L = attn::PrefillLayout<D, PAGED, FP8, SPARSE>;
  auto kernel = attn::prefill_fwd_kernel<D, CAUSAL, WINDOW, PAGED, FP8, SPARSE, BIAS>;
  cudaError_t e =
      ensure_smem_limit<attn::prefill_fwd_kernel<D, CAUSAL, WINDOW, PAGED, FP8, SPARSE, BIAS>>(L::kAlloc);
  if (e != cudaSuccess) return fail_cuda(e);
  const int sms = sm_count();
  if (sms <= 0) return fail_cuda(cudaErrorInvalidDevice);
  // Persistent: one CTA per SM (or per work item when there are fewer; the
  // paged kernels count their items on the device and always take one per SM).
  const unsigned grid = static_cast<unsigned>(PAGED || p.num_items >= sms ? sms : p.num_items);
  kernel<<<grid, attn::kPrefillThreads, L::kAlloc, stream>>>(tq, tk, tv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail_cuda(e);
  return ATTN_OK;
}

int decode_heads_per_cta(int Hkv) {
  int hb = 1;
  while (hb < 8 && Hkv % (hb * 2) == 0) hb *= 2;
  return hb;
}

// The split plan depends only on sizes (the lengths live on the device): 256
// tokens per split, halved (down to 64) while a full-length batch would give
// fewer than kDecodeTargetCtas CTAs, so small batches still fill the GPU.
constexpr long long kDecodeTargetCtas = 2 * 148;

int split_tokens_for(int num_seqs, int Hkv, int max_pages, int page_size) {
  (void)Hkv;
  const long long max_tokens = static_cast<long long>(max_pages) * page_size;
  long long split = 256;
  while (split > 64 && num_seqs * ((max_tokens + split - 1) / split) < kDecodeTargetCtas) split /= 2;
  return static_cast<int>(split);
}

// KV heads per CTA: up to 8 (one page chunk of all heads per TMA box pair),
// fewer when that leaves too few CTAs.
int decode_heads_for(int num_seqs, int Hkv, int max_splits) {
  int hb = decode_heads_per_cta(Hkv);
  while (hb > 1 && static_cast<long long>(num_seqs) * max_splits * (Hkv / hb) < kDecodeTargetCtas) hb /= 2;
  return hb;
}

struct DecodePlan {
  int split_tokens = 0;
  int max_splits = 0;
  size_t o_bytes = 0;
  size_t lse_offset = 0;
  size_t total = 0;
};

bool decode_plan(int num_seqs, int Hq, int Hkv, int d, int max_pages, int page_size, DecodePlan* out) {
  if (num_seqs < 1 || Hq < 1 || max_pages < 1 || page_size < 1 || (d != 64 && d != 128)) return false;
  const long long max_tokens = static_cast<long long>(max_pages) * page_size;
  if (max_tokens > INT_MAX) return false;
  DecodePlan pl;
  pl.split_tokens = split_tokens_for(num_seqs, Hkv, max_pages, page_size);
  pl.max_splits = static_cast<int>((max_tokens + pl.split_tokens - 1) / pl.split_tokens);
  const size_t rows = static_cast<size_t>(num_seqs) * Hq * pl.max_splits;
  pl.o_bytes = rows * d * sizeof(float);
  pl.lse_offset = (pl.o_bytes + 255) & ~static_cast<size_t>(255);
  pl.total = pl.lse_offset + rows * sizeof(float);
  *out = pl;
  return true;
}

template <int D, int HB>
int launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const attn::DecodeParams& p,
                  attn_bf16* o, float* lse, cudaStream_t stream) {
  using L = attn::DecodeLayout<D, HB>;
  auto split_kernel = attn::decode_split_kernel<D, HB>;
  cudaError_t e = ensure_smem_limit<attn::decode_split_kernel<D, HB>>(L::kAlloc);
  if (e != cudaSuccess) return fail_cuda(e);
  const dim3 grid(static_cast<unsigned>(p.max_splits), static_cast<unsigned>(p.S),
                  static_cast<unsigned>(p.Hkv / HB));
  split_kernel<<<grid, 32 * (HB + 1), L::kAlloc, stream>>>(tk, tv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail_cuda(e);
  const long long warps = static_cast<long long>(p.S) * p.Hq;
  const unsigned mgrid = static_cast<unsigned>((warps * 32 + attn::kMergeThreads - 1) / attn::kMergeThreads);
  // The merge may launch while the split pass's last wave runs (see
  // decode_split_kernel); it waits for the split grid in griddepcontrol.wait.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mgrid);
  cfg.blockDim = dim3(attn::kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, attn::decode_merge_kernel<D>, p, reinterpret_cast<__nv_bfloat16*>(o), lse);
  if (e != cudaSuccess) return fail_cuda(e);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail_cuda(e);
  return ATTN_OK;
}

template <int D>
int dispatch_decode_hb(int hb, const CUtensorMap& tk, const CUtensorMap& tv,
                       const attn::DecodeParams& p, attn_bf16* o, float* lse, cudaStream_t stream) {
  switch (hb) {
    case 8: return launch_decode<D, 8>(tk, tv, p, o, lse, stream);
    case 4: return launch_decode<D, 4>(tk, tv, p, o, lse, stream);
    case 2: return launch_decode<D, 2>(tk, tv, p, o, lse, stream);
    default: return launch_decode<D, 1>(tk, tv, p, o, lse, stream);
  }
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return 1; }

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_NULL: return "a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "a size is out of range or inconsistent";
    case ATTN_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_ERR_UNSUPPORTED: return "input valid but not supported by this build";
    case ATTN_ERR_LAUNCH: return "CUDA refused the launch";
    case ATTN_ERR_DEVICE: return "a kernel recorded a runtime error";
    default: return "unknown status";
  }
}

int attn_last_cuda_error(void) { return t_last_cuda_error; }

int attn_fwd_window(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse,
                    int B, int Hq, int Hkv, int N, int d, int causal, int window_left, float scale,
                    void* stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  if (causal != 0 && causal != 1) return ATTN_ERR_SHAPE;
  if (window_left < -1) return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_SHAPE;
  const long long bh = static_cast<long long>(B) * Hq;
  const long long blocks = (static_cast<long long>(N) + 255) / 256;
  if (bh > INT_MAX || blocks * bh > INT_MAX) return ATTN_ERR_SHAPE;
  if (misaligned16(q) || misaligned16(k) || misaligned16(v) || misaligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_ALIGN;

  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = static_cast<uint64_t>(d) * 2;
  const uint64_t head_bytes = row_bytes * static_cast<uint64_t>(N);
  if (!encode_3d(&tq, q, d, N, static_cast<uint64_t>(B) * Hq, row_bytes, head_bytes, 64, 128, 1) ||
      !encode_3d(&tk, k, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 64, 128, 1) ||
      !encode_3d(&tv, v, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 64, 128, 1))
    return fail_cuda(cudaErrorInvalidValue);

  attn::PrefillParams p;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.num_m = static_cast<int>(blocks);
  p.num_items = static_cast<int>(blocks * bh);
  p.window_left = window_left >= N - 1 ? -1 : window_left;  // a window covering every key is no window
  p.scale_log2 = scale * kLog2e;
  p.o_scale = 1.f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool win = p.window_left >= 0;
  if (d == 128) {
    if (win)
      return causal ? launch_prefill<128, true, true>(tq, tk, tv, p, s) : launch_prefill<128, false, true>(tq, tk, tv, p, s);
    return causal ? launch_prefill<128, true, false>(tq, tk, tv, p, s) : launch_prefill<128, false, false>(tq, tk, tv, p, s);
  }
  if (win)
    return causal ? launch_prefill<64, true, true>(tq, tk, tv, p, s) : launch_prefill<64, false, true>(tq, tk, tv, p, s);
  return causal ? launch_prefill<64, true, false>(tq, tk, tv, p, s) : launch_prefill<64, false, false>(tq, tk, tv, p, s);
}

int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B,
             int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  return attn_fwd_window(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, -1, scale, stream);
}

int paged_attn_decode_split_tokens(int num_seqs, int Hkv, int max_pages, int page_size) {
  return split_tokens_for(num_seqs, Hkv, max_pages, page_size);
}

size_t paged_attn_decode_workspace_bytes(int num_seqs, int Hq, int d, int max_pages, int page_size) {
  DecodePlan pl;
  if (!decode_plan(num_seqs, Hq, 1, d, max_pages, page_size, &pl)) return 0;
  return pl.total;
}

}  // extern "C"

namespace {

// Host-side argument checks of paged_attn_decode (no CUDA call).
int validate_decode(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                    const int32_t* block_table, const int32_t* seq_lens, int page_size, attn_bf16* o,
                    float* lse, int num_seqs, int Hq, int Hkv, int d, int max_pages, int num_pages,
                    float scale, void* workspace, size_t workspace_bytes, DecodePlan* plan) {
  if (!q || !k_pool || !v_pool || !block_table || !seq_lens || !o || !lse) return ATTN_ERR_NULL;
  if (num_seqs < 1 || Hq < 1 || Hkv < 1 || max_pages < 1 || num_pages < 1 || page_size < 1)
    return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_SHAPE;
  if (num_seqs > 65535 || Hkv > 65535) return ATTN_ERR_SHAPE;
  if (static_cast<long long>(num_pages) * page_size > INT_MAX) return ATTN_ERR_SHAPE;
  if (page_size % 16 != 0 || page_size > 256) return ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 16) return ATTN_ERR_UNSUPPORTED;
  DecodePlan pl;
  if (!decode_plan(num_seqs, Hq, Hkv, d, max_pages, page_size, &pl)) return ATTN_ERR_SHAPE;
  if (!workspace) return ATTN_ERR_WORKSPACE;
  if (workspace_bytes < pl.total) return ATTN_ERR_WORKSPACE;
  if (misaligned16(q) || misaligned16(k_pool) || misaligned16(v_pool) || misaligned16(o) ||
      misaligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) != 0)
    return ATTN_ERR_ALIGN;
  *plan = pl;
  return ATTN_OK;
}

}  // namespace

// Library-internal (hidden, not part of the C ABI): used by the no-alloc
// entry point in attn_noalloc.cu, which is built as a separate file.
// attn_internal_validate_decode runs paged_attn_decode's host-side checks
// (no CUDA call); attn_internal_cuda_failure records a CUDA error for
// attn_last_cuda_error and returns ATTN_ERR_LAUNCH.
__attribute__((visibility("hidden"))) int attn_internal_validate_decode(
    const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool, const int32_t* block_table,
    const int32_t* seq_lens, int page_size, attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
    int max_pages, int num_pages, float scale, void* workspace, size_t workspace_bytes) {
  DecodePlan pl;
  return validate_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv, d,
                         max_pages, num_pages, scale, workspace, workspace_bytes, &pl);
}

__attribute__((visibility("hidden"))) int attn_internal_cuda_failure(cudaError_t e) { return fail_cuda(e); }

extern "C" {


int paged_attn_decode(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                      const int32_t* block_table, const int32_t* seq_lens, int page_size,
                      attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
                      int max_pages, int num_pages, float scale, void* workspace,
                      size_t workspace_bytes, void* stream) {
  DecodePlan pl;
  const int vs = validate_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv,
                                 d, max_pages, num_pages, scale, workspace, workspace_bytes, &pl);
  if (vs != ATTN_OK) return vs;

  const int hb = decode_heads_for(num_seqs, Hkv, pl.max_splits);
  CUtensorMap tk, tv;
  const uint64_t token_bytes = static_cast<uint64_t>(Hkv) * d * 2;
  const uint64_t head_bytes = static_cast<uint64_t>(d) * 2;
  const uint64_t rows = static_cast<uint64_t>(num_pages) * page_size;
  if (!encode_3d(&tk, k_pool, d, rows, Hkv, token_bytes, head_bytes, 64, attn::kDecodeChunk, hb) ||
      !encode_3d(&tv, v_pool, d, rows, Hkv, token_bytes, head_bytes, 64, attn::kDecodeChunk, hb))
    return fail_cuda(cudaErrorInvalidValue);

  attn::DecodeParams p;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.lse_offset);
  p.S = num_seqs;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.page_size = page_size;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.max_splits = pl.max_splits;
  p.split_tokens = pl.split_tokens;
  p.scale_log2 = scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128) return dispatch_decode_hb<128>(hb, tk, tv, p, o, lse, s);
  return dispatch_decode_hb<64>(hb, tk, tv, p, o, lse, s);
}

}  // extern "C"

// A captured decode step: the split pass and the merge as one CUDA graph.
struct attn_decode_graph {
  cudaGraphExec_t exec = nullptr;
  int device = -1;
};

namespace {

// Everything a decode launch needs that is not a stream operation, done
// before capture so that capture only records the two kernel launches.
cudaError_t prepare_decode(int d, int Hkv, int num_seqs, int max_splits) {
  if (!encode_fn()) return cudaErrorInvalidValue;
  const int hb = decode_heads_for(num_seqs, Hkv, max_splits);
  auto one = [&](auto tag) -> cudaError_t {
    constexpr int D = decltype(tag)::value;
    switch (hb) {
      case 8: return ensure_smem_limit<attn::decode_split_kernel<D, 8>>(attn::DecodeLayout<D, 8>::kAlloc);
      case 4: return ensure_smem_limit<attn::decode_split_kernel<D, 4>>(attn::DecodeLayout<D, 4>::kAlloc);
      case 2: return ensure_smem_limit<attn::decode_split_kernel<D, 2>>(attn::DecodeLayout<D, 2>::kAlloc);
      default: return ensure_smem_limit<attn::decode_split_kernel<D, 1>>(attn::DecodeLayout<D, 1>::kAlloc);
    }
  };
  return d == 128 ? one(std::integral_constant<int, 128>{}) : one(std::integral_constant<int, 64>{});
}

}  // namespace

extern "C" {

int paged_attn_decode_graph_create(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                                   const int32_t* block_table, const int32_t* seq_lens, int page_size,
                                   attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
                                   int max_pages, int num_pages, float scale, void* workspace,
                                   size_t workspace_bytes, attn_decode_graph** graph) {
  if (!graph) return ATTN_ERR_NULL;
  *graph = nullptr;
  DecodePlan pl;
  const int vs = validate_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv,
                                 d, max_pages, num_pages, scale, workspace, workspace_bytes, &pl);
  if (vs != ATTN_OK) return vs;
  {
    const cudaError_t e = prepare_decode(d, Hkv, num_seqs, pl.max_splits);
    if (e != cudaSuccess) return fail_cuda(e);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  cudaStream_t s = nullptr;
  e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e != cudaSuccess) return fail_cuda(e);
  e = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) {
    cudaStreamDestroy(s);
    return fail_cuda(e);
  }
  const int rc = paged_attn_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq,
                                   Hkv, d, max_pages, num_pages, scale, workspace, workspace_bytes, s);
  cudaGraph_t g = nullptr;
  const cudaError_t end = cudaStreamEndCapture(s, &g);
  cudaStreamDestroy(s);
  if (rc != ATTN_OK || end != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return rc != ATTN_OK ? rc : fail_cuda(end);
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, g, 0);
  cudaGraphDestroy(g);
  if (e != cudaSuccess) return fail_cuda(e);
  attn_decode_graph* h = new (std::nothrow) attn_decode_graph;
  if (!h) {
    cudaGraphExecDestroy(exec);
    return fail_cuda(cudaErrorMemoryAllocation);
  }
  h->exec = exec;
  h->device = dev;
  *graph = h;
  return ATTN_OK;
}

int paged_attn_decode_graph_launch(attn_decode_graph* graph, void* stream) {
  if (!graph || !graph->exec) return ATTN_ERR_NULL;
  const cudaError_t e = cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  return ATTN_OK;
}

int paged_attn_decode_graph_destroy(attn_decode_graph* graph) {
  if (!graph) return ATTN_OK;
  cudaError_t e = cudaSuccess;
  if (graph->exec) e = cudaGraphExecDestroy(graph->exec);
  delete graph;
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e);
}

int attn_device_status(void* stream, unsigned int* bits) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, attn::g_attn_device_error, sizeof(word));
  if (e != cudaSuccess) return fail_cuda(e);
  if (bits) *bits = word;
  if (word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(attn::g_attn_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail_cuda(e);
    return ATTN_ERR_DEVICE;
  }
  return ATTN_OK;
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Appending to a paged cache, and chunked prefill over it
// ----------------------------------------------------------------------------

namespace {

bool page_size_supported(int page_size) {
  return page_size == 16 || page_size == 32 || page_size == 64 || page_size == 128 || page_size == 256;
}

bool misaligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) != 0; }

// Checks shared by the append and the chunked prefill (no CUDA call).
int validate_paged_cache(const void* k_pool, const void* v_pool, const int32_t* cu_seqlens_q,
                         const int32_t* seq_lens, const int32_t* block_table, int num_seqs, int total_q, int Hkv,
                         int d, int page_size, int max_pages, int num_pages) {
  if (!k_pool || !v_pool || !cu_seqlens_q || !seq_lens || !block_table) return ATTN_ERR_NULL;
  if (num_seqs < 1 || total_q < 0 || Hkv < 1 || max_pages < 1 || num_pages < 1 || page_size < 1)
    return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_SHAPE;
  if (Hkv > 65535) return ATTN_ERR_SHAPE;
  if (static_cast<long long>(num_pages) * page_size > INT_MAX ||
      static_cast<long long>(max_pages) * page_size > INT_MAX ||
      static_cast<long long>(num_seqs) * max_pages > INT_MAX)
    return ATTN_ERR_SHAPE;
  if (!page_size_supported(page_size)) return ATTN_ERR_UNSUPPORTED;
  if (misaligned16(k_pool) || misaligned16(v_pool) || misaligned4(cu_seqlens_q) || misaligned4(seq_lens) ||
      misaligned4(block_table))
    return ATTN_ERR_ALIGN;
  return ATTN_OK;
}

int validate_paged_prefill(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                           const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table,
                           attn_bf16* o, float* lse, int num_seqs, int total_q, int Hq, int Hkv, int d,
                           int page_size, int max_pages, int num_pages, int causal, float scale) {
  if (!q || !o || !lse) return ATTN_ERR_NULL;
  const int st = validate_paged_cache(k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, num_seqs, total_q, Hkv,
                                      d, page_size, max_pages, num_pages);
  if (st != ATTN_OK) return st;
  if (Hq < 1 || Hq % Hkv != 0 || Hq > 65535) return ATTN_ERR_SHAPE;
  if (causal != 0 && causal != 1) return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_SHAPE;
  if (static_cast<long long>(total_q) * Hq > INT_MAX) return ATTN_ERR_SHAPE;
  if (num_seqs > attn::kPagedMaxSeqs) return ATTN_ERR_UNSUPPORTED;
  // Query blocks of 256 rows: at most ceil(q_len / 256) per sequence.
  if ((static_cast<long long>(total_q) + 255LL * num_seqs) / 256 > attn::kPagedMaxBlocks) return ATTN_ERR_UNSUPPORTED;
  if (misaligned16(q) || misaligned16(o) || misaligned4(lse)) return ATTN_ERR_ALIGN;
  return ATTN_OK;
}

int launch_append(const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_pool, attn_bf16* v_pool,
                  const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table, int num_seqs,
                  int total_q, int Hkv, int d, int page_size, int max_pages, int num_pages, cudaStream_t stream) {
  if (total_q == 0) return ATTN_OK;
  const int sms = sm_count();
  if (sms <= 0) return fail_cuda(cudaErrorInvalidDevice);
  attn::AppendParams p;
  p.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
  p.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
  p.k_pool = reinterpret_cast<__nv_bfloat16*>(k_pool);
  p.v_pool = reinterpret_cast<__nv_bfloat16*>(v_pool);
  p.cu_q = cu_seqlens_q;
  p.seq_lens = seq_lens;
  p.block_table = block_table;
  p.num_seqs = num_seqs;
  p.total_q = total_q;
  p.Hkv = Hkv;
  p.D = d;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.page_size = page_size;
  // One warp per kAppendTokensPerWarp consecutive new tokens.
  constexpr long long kTokensPerBlock = attn::kAppendThreads / 32 * attn::kAppendTokensPerWarp;
  const unsigned grid = static_cast<unsigned>((static_cast<long long>(total_q) + kTokensPerBlock - 1) / kTokensPerBlock);
  attn::paged_append_kernel<<<grid, attn::kAppendThreads, 0, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e);
}

int launch_paged_prefill(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                         const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table,
                         attn_bf16* o, float* lse, int num_seqs, int total_q, int Hq, int Hkv, int d, int page_size,
                         int max_pages, int num_pages, int causal, float scale, cudaStream_t stream) {
  if (total_q == 0) return ATTN_OK;
  const int box_rows = page_size < 128 ? page_size : 128;
  CUtensorMap tq, tk, tv;
  const uint64_t d2 = static_cast<uint64_t>(d) * 2;
  // Q: (d, packed token, head); pools: (d, page * page_size + slot, kv head).
  if (!encode_3d(&tq, q, d, static_cast<uint64_t>(total_q), Hq, static_cast<uint64_t>(Hq) * d2, d2, 64, 128, 1) ||
      !encode_3d(&tk, k_pool, d, static_cast<uint64_t>(num_pages) * page_size, Hkv, static_cast<uint64_t>(Hkv) * d2,
                 d2, 64, static_cast<uint32_t>(box_rows), 1) ||
      !encode_3d(&tv, v_pool, d, static_cast<uint64_t>(num_pages) * page_size, Hkv, static_cast<uint64_t>(Hkv) * d2,
                 d2, 64, static_cast<uint32_t>(box_rows), 1))
    return fail_cuda(cudaErrorInvalidValue);
  attn::PrefillParams p{};
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = 1;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = 0;
  p.group = Hq / Hkv;
  p.num_m = 0;
  p.num_items = 0;
  p.window_left = -1;
  p.scale_log2 = scale * kLog2e;
  p.o_scale = 1.f;
  p.cu_q = cu_seqlens_q;
  p.seq_lens = seq_lens;
  p.block_table = block_table;
  p.k_pool = reinterpret_cast<const __nv_bfloat16*>(k_pool);
  p.v_pool = reinterpret_cast<const __nv_bfloat16*>(v_pool);
  p.num_seqs = num_seqs;
  p.total_q = total_q;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.page_size = page_size;
  p.page_box = box_rows;
  if (d == 128)
    return causal ? launch_prefill<128, true, false, true>(tq, tk, tv, p, stream)
                  : launch_prefill<128, false, false, true>(tq, tk, tv, p, stream);
  return causal ? launch_prefill<64, true, false, true>(tq, tk, tv, p, stream)
                : launch_prefill<64, false, false, true>(tq, tk, tv, p, stream);
}

}  // namespace

extern "C" {

int paged_kv_append(const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_pool, attn_bf16* v_pool,
                    const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table, int num_seqs,
                    int total_q, int Hkv, int d, int page_size, int max_pages, int num_pages, void* stream) {
  const int st = validate_paged_cache(k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, num_seqs, total_q, Hkv,
                                      d, page_size, max_pages, num_pages);
  if (st != ATTN_OK) return st;
  if (total_q > 0 && (!k_new || !v_new)) return ATTN_ERR_NULL;
  if (total_q > 0 && (misaligned16(k_new) || misaligned16(v_new))) return ATTN_ERR_ALIGN;
  return launch_append(k_new, v_new, k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, num_seqs, total_q, Hkv, d,
                       page_size, max_pages, num_pages, static_cast<cudaStream_t>(stream));
}

int paged_prefill(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                  const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table, attn_bf16* o,
                  float* lse, int num_seqs, int total_q, int Hq, int Hkv, int d, int page_size, int max_pages,
                  int num_pages, int causal, float scale, void* stream) {
  const int st = validate_paged_prefill(q, k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, o, lse, num_seqs,
                                        total_q, Hq, Hkv, d, page_size, max_pages, num_pages, causal, scale);
  if (st != ATTN_OK) return st;
  return launch_paged_prefill(q, k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, o, lse, num_seqs, total_q, Hq,
                              Hkv, d, page_size, max_pages, num_pages, causal, scale,
                              static_cast<cudaStream_t>(stream));
}

int paged_prefill_append(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_pool,
                         attn_bf16* v_pool, const int32_t* cu_seqlens_q, const int32_t* seq_lens,
                         const int32_t* block_table, attn_bf16* o, float* lse, int num_seqs, int total_q, int Hq,
                         int Hkv, int d, int page_size, int max_pages, int num_pages, int causal, float scale,
                         void* stream) {
  const int st = validate_paged_prefill(q, k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, o, lse, num_seqs,
                                        total_q, Hq, Hkv, d, page_size, max_pages, num_pages, causal, scale);
  if (st != ATTN_OK) return st;
  if (total_q > 0 && (!k_new || !v_new)) return ATTN_ERR_NULL;
  if (total_q > 0 && (misaligned16(k_new) || misaligned16(v_new))) return ATTN_ERR_ALIGN;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int a = launch_append(k_new, v_new, k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, num_seqs, total_q,
                              Hkv, d, page_size, max_pages, num_pages, s);
  if (a != ATTN_OK) return a;
  return launch_paged_prefill(q, k_pool, v_pool, cu_seqlens_q, seq_lens, block_table, o, lse, num_seqs, total_q, Hq,
                              Hkv, d, page_size, max_pages, num_pages, causal, scale, s);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// FP8 (e4m3) prefill
// ----------------------------------------------------------------------------

extern "C" {

int attn_fwd_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v, attn_bf16* o, float* lse, int B, int Hq,
                 int Hkv, int N, int d, int causal, float scale, float q_descale, float k_descale, float v_descale,
                 void* stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  if (causal != 0 && causal != 1) return ATTN_ERR_SHAPE;
  for (const float x : {scale, q_descale, k_descale, v_descale})
    if (!(x > 0.f) || !std::isfinite(x)) return ATTN_ERR_SHAPE;
  if (!std::isfinite(scale * q_descale * k_descale * kLog2e)) return ATTN_ERR_SHAPE;
  const long long bh = static_cast<long long>(B) * Hq;
  const long long blocks = (static_cast<long long>(N) + 255) / 256;
  if (bh > INT_MAX || blocks * bh > INT_MAX) return ATTN_ERR_SHAPE;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;  // an e4m3 row of 128 is exactly one 128-byte swizzled box
  if (misaligned16(q) || misaligned16(k) || misaligned16(v) || misaligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return ATTN_ERR_ALIGN;

  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = static_cast<uint64_t>(d);  // one byte per element
  const uint64_t head_bytes = row_bytes * static_cast<uint64_t>(N);
  if (!encode_3d(&tq, q, d, N, static_cast<uint64_t>(B) * Hq, row_bytes, head_bytes, 128, 128, 1,
                 CU_TENSOR_MAP_DATA_TYPE_UINT8) ||
      !encode_3d(&tk, k, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 128, 128, 1,
                 CU_TENSOR_MAP_DATA_TYPE_UINT8) ||
      !encode_3d(&tv, v, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 128, 128, 1,
                 CU_TENSOR_MAP_DATA_TYPE_UINT8))
    return fail_cuda(cudaErrorInvalidValue);

  attn::PrefillParams p{};
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.num_m = static_cast<int>(blocks);
  p.num_items = static_cast<int>(blocks * bh);
  p.window_left = -1;
  p.scale_log2 = scale * q_descale * k_descale * kLog2e;
  p.o_scale = v_descale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return causal ? launch_prefill<128, true, false, false, true>(tq, tk, tv, p, s)
                : launch_prefill<128, false, false, false, true>(tq, tk, tv, p, s);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Block-sparse prefill
// ----------------------------------------------------------------------------

extern "C" {

int attn_fwd_block_sparse(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse,
                          int B, int Hq, int Hkv, int N, int d, int causal, float scale, const uint64_t* block_mask,
                          long long mask_b_stride, long long mask_h_stride, void* stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return ATTN_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  if (causal != 0 && causal != 1) return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_SHAPE;
  if (mask_b_stride < 0 || mask_h_stride < 0) return ATTN_ERR_SHAPE;
  const long long bh = static_cast<long long>(B) * Hq;
  const long long blocks = (static_cast<long long>(N) + 255) / 256;
  if (bh > INT_MAX || blocks * bh > INT_MAX) return ATTN_ERR_SHAPE;
  const int kv_tiles = (N + 127) / 128;
  const int words = (kv_tiles + 63) / 64;
  if (words > attn::kMaskWords) return ATTN_ERR_UNSUPPORTED;  // N <= 32768
  if (misaligned16(q) || misaligned16(k) || misaligned16(v) || misaligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 || (reinterpret_cast<uintptr_t>(block_mask) & 7u) != 0)
    return ATTN_ERR_ALIGN;

  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = static_cast<uint64_t>(d) * 2;
  const uint64_t head_bytes = row_bytes * static_cast<uint64_t>(N);
  if (!encode_3d(&tq, q, d, N, static_cast<uint64_t>(B) * Hq, row_bytes, head_bytes, 64, 128, 1) ||
      !encode_3d(&tk, k, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 64, 128, 1) ||
      !encode_3d(&tv, v, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 64, 128, 1))
    return fail_cuda(cudaErrorInvalidValue);

  attn::PrefillParams p{};
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.num_m = static_cast<int>(blocks);
  p.num_items = static_cast<int>(blocks * bh);
  p.window_left = -1;
  p.scale_log2 = scale * kLog2e;
  p.o_scale = 1.f;
  p.block_mask = block_mask;
  p.mask_b_stride = mask_b_stride;
  p.mask_h_stride = mask_h_stride;
  p.mask_words = words;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_prefill<128, true, false, false, false, true>(tq, tk, tv, p, s)
                  : launch_prefill<128, false, false, false, false, true>(tq, tk, tv, p, s);
  return causal ? launch_prefill<64, true, false, false, false, true>(tq, tk, tv, p, s)
                : launch_prefill<64, false, false, false, false, true>(tq, tk, tv, p, s);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Additive M
// ----------------------------------------------------------------------------

extern "C" {

int attn_fwd_bias(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B,
                  int Hq, int Hkv, int N, int d, int causal, float scale, const attn_bf16* bias,
                  long long bias_b_stride, long long bias_h_stride, long long bias_row_stride, void* stream) {
  if (!q || !k || !v || !o || !lse || !bias) return ATTN_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_SHAPE;
  if (d != 64 && d != 128) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
  if (causal != 0 && causal != 1) return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_SHAPE;
  if (bias_b_stride < 0 || bias_h_stride < 0 || bias_row_stride < 0) return ATTN_ERR_SHAPE;
  const long long padded = (static_cast<long long>(N) + 7) / 8 * 8;
  if (bias_row_stride != 0 && bias_row_stride < padded) return ATTN_ERR_SHAPE;  // rows hold N (padded) values
  const long long bh = static_cast<long long>(B) * Hq;
  const long long blocks = (static_cast<long long>(N) + 255) / 256;
  if (bh > INT_MAX || blocks * bh > INT_MAX) return ATTN_ERR_SHAPE;
  if (misaligned16(q) || misaligned16(k) || misaligned16(v) || misaligned16(o) || misaligned16(bias) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 || bias_b_stride % 8 != 0 || bias_h_stride % 8 != 0 ||
      bias_row_stride % 8 != 0)
    return ATTN_ERR_ALIGN;

  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = static_cast<uint64_t>(d) * 2;
  const uint64_t head_bytes = row_bytes * static_cast<uint64_t>(N);
  if (!encode_3d(&tq, q, d, N, static_cast<uint64_t>(B) * Hq, row_bytes, head_bytes, 64, 128, 1) ||
      !encode_3d(&tk, k, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 64, 128, 1) ||
      !encode_3d(&tv, v, d, N, static_cast<uint64_t>(B) * Hkv, row_bytes, head_bytes, 64, 128, 1))
    return fail_cuda(cudaErrorInvalidValue);

  attn::PrefillParams p{};
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  p.num_m = static_cast<int>(blocks);
  p.num_items = static_cast<int>(blocks * bh);
  p.window_left = -1;
  p.scale_log2 = scale * kLog2e;
  p.scale = scale;
  p.o_scale = 1.f;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  p.bias_b_stride = bias_b_stride;
  p.bias_h_stride = bias_h_stride;
  p.bias_row_stride = bias_row_stride;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_prefill<128, true, false, false, false, false, true>(tq, tk, tv, p, s)
                  : launch_prefill<128, false, false, false, false, false, true>(tq, tk, tv, p, s);
  return causal ? launch_prefill<64, true, false, false, false, false, true>(tq, tk, tv, p, s)
                : launch_prefill<64, false, false, false, false, false, true>(tq, tk, tv, p, s);
}

}  // extern "C"

