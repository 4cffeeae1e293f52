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
// exits.  It comes into being when the CUDA runtime loads this library's
// device code on a device; with lazy module loading (the default since CUDA
// 12.2) that is the first call here on that device, so that call can fail
// with ATTN_ERR_LAUNCH (attn_last_cuda_error() then names the CUDA error,
// e.g. out of memory) when the device is already full.  A warm-up call at
// start-up settles this once.
//
// In host code the array's name is only a host-side stand-in, never a device
// address: the address a kernel may use is fetched with cudaGetSymbolAddress
// once per CUDA context, with that context current, and cached under the
// context's unique id, so a device reset (which gives the device a new
// context and a new copy of the array) is followed by a fresh lookup.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "attn_b200.h"

// Host-side checks of paged_attn_decode and CUDA error recording, defined in
// attn_api.cu (hidden, not part of the C ABI).
int attn_internal_validate_decode(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                                  const int32_t* block_table, const int32_t* seq_lens, int page_size,
                                  attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
                                  int max_pages, int num_pages, float scale, void* workspace,
                                  size_t workspace_bytes);
int attn_internal_cuda_failure(cudaError_t e);

namespace {

static_assert(ATTN_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const DriverFns& driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

// Unique id of the calling thread's current CUDA context; false when there is
// none yet (the runtime creates it on first use) or it cannot be queried.
bool current_context_id(unsigned long long* id) {
  const DriverFns& f = driver_fns();
  if (!f.get_current || !f.get_id) return false;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return f.get_id(ctx, id) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  bool valid = false;
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
std::mutex g_setup_mutex;
ScratchSlot g_slots[kMaxDevices];

// Device address of the scratch array in the current device's context: looked
// up (cudaGetSymbolAddress) on the first call in each context and cached under
// the context id.  Without a context id (none current yet, or the driver
// cannot report one) the address is looked up afresh and not cached.
int scratch_for_current_context(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return attn_internal_cuda_failure(e);
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  ScratchSlot& slot = g_slots[dev];
  if (have_id && slot.valid && slot.ctx_id == id) {
    *out = slot.ptr;
    return ATTN_OK;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return attn_internal_cuda_failure(e);
  if (p == nullptr) return ATTN_ERR_LAUNCH;
  // The lookup may have created the context: ask for its id again.
  slot.valid = current_context_id(&id);
  slot.ctx_id = id;
  slot.ptr = p;
  *out = p;
  return ATTN_OK;
}

}  // namespace

extern "C" int paged_attn_decode_noalloc(const attn_bf16* q, const attn_bf16* k_pool,
                                         const attn_bf16* v_pool, const int32_t* block_table,
                                         const int32_t* seq_lens, int page_size, attn_bf16* o,
                                         float* lse, int num_seqs, int Hq, int Hkv, int d,
                                         int max_pages, int num_pages, float scale, void* stream) {
  // paged_attn_decode's own checks first, before any CUDA call, with a
  // stand-in workspace of unbounded size (non-null, aligned, never
  // dereferenced), so a bad argument is reported as itself; only then is the
  // problem's scratch need compared with the array.
  void* const stand_in = reinterpret_cast<void*>(static_cast<uintptr_t>(256));
  const int vs = attn_internal_validate_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse,
                                               num_seqs, Hq, Hkv, d, max_pages, num_pages, scale, stand_in,
                                               SIZE_MAX);
  if (vs != ATTN_OK) return vs;
  if (paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_pages, page_size) > ATTN_NOALLOC_SCRATCH_BYTES)
    return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_for_current_context(&scratch);
  if (rc != ATTN_OK) return rc;
  return paged_attn_decode(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv, d,
                           max_pages, num_pages, scale, scratch, ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
