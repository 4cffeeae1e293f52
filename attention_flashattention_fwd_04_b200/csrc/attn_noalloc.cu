// paged_attn_decode_noalloc: the paged decode for callers that may not
// allocate device memory.
//
// Some callers cannot hand us a workspace: a plug-in whose host program owns
// every byte of device memory and forbids its plug-ins to allocate, a
// latency-critical serving loop where a cudaMalloc could synchronise the
// device and stall every other stream, or a process whose caching allocator
// has already reserved all free memory.  For them the split partials live in
// a fixed array compiled into this library instead of a caller buffer.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library's device code is loaded holds its full size until the process
// exits.  In host code the array's name is only a host-side stand-in, never a
// device address: the address a kernel may use is fetched once per device
// with cudaGetSymbolAddress.
#include <cuda_runtime.h>

#include <mutex>

#include "attn_b200.h"

namespace {

static_assert(ATTN_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device; looked up on the
// first call made with that device current.
int scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return ATTN_ERR_LAUNCH;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" int paged_attn_decode_noalloc(const attn_bf16* q, const attn_bf16* k_pool,
                                         const attn_bf16* v_pool, const int32_t* block_table,
                                         const int32_t* seq_lens, int page_size, attn_bf16* o,
                                         float* lse, int num_seqs, int Hq, int Hkv, int d,
                                         int max_pages, int num_pages, float scale, void* stream) {
  // Argument and size checks first, so a bad or oversized call is refused
  // before any CUDA call.
  if (!q || !k_pool || !v_pool || !block_table || !seq_lens || !o || !lse) return ATTN_ERR_NULL;
  const size_t need = paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_pages, page_size);
  if (need > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const int rc = scratch_for_current_device(&scratch);
    if (rc != ATTN_OK) return rc;
  }
  // need == 0 means the sizes are invalid: the regular entry point reports
  // which argument is wrong (a NULL workspace is only blamed last).
  return paged_attn_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq,
                           Hkv, d, max_pages, num_pages, scale, scratch, ATTN_NOALLOC_SCRATCH_BYTES,
                           stream);
}
