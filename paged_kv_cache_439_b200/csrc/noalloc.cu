// pkv_paged_attention_decode_noalloc: the decode entry point for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain device memory for the split-K scratch:
// code embedded in a host runtime that owns every device allocation and hands
// its plugins no allocator or workspace, or latency-critical paths where an
// allocation (and the device synchronisation cudaMalloc/cudaFree can imply)
// is not acceptable.  This entry point takes the same inputs and outputs as
// pkv_paged_attention_decode but keeps the split-K scratch in one fixed device
// array that lives inside this library.
//
// Properties a caller has to know:
//  * The array holds PKV_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads
//    the library, until the process exits.
//  * Shapes whose split-K scratch (pkv_workspace_size) exceeds it are rejected
//    with PKV_ERR_SCRATCH_LIMIT before anything is launched.
//  * All calls share the array.  Calls whose kernels overlap on the GPU (for
//    example on two streams) race on it; serialise them.
//  * The array keeps whatever the previous call left.  Nothing has to start at
//    zero: every scratch entry the merge kernel reads is first written by the
//    decode kernel of the same call.
//  * The first call in each CUDA context (normally once per device, the
//    device's primary context) looks up the array's device address
//    (cudaGetSymbolAddress, with that device current) and caches it together
//    with the context's unique id.  A later call in another context (after a
//    cudaDeviceReset, for example, which makes the module load again and can
//    move the array) looks the address up afresh instead of reusing it.
//  * The driver reserves the array's 16 MiB when it loads the module that
//    holds it.  With lazy module loading (the CUDA default) that happens at
//    this first call, which can therefore fail with PKV_ERR_CUDA when the
//    device has no 16 MiB left.  Make the first call at start-up, before any
//    stream capture.
//  * Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pkv.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchSlot {
  unsigned long long ctx_id;  // unique id of the context the address belongs to
  void* addr;                 // device address of g_decode_scratch in that context
};
ScratchSlot g_scratch[kMaxDevices];

// cuCtxGetId (unique per context for the life of the process, never reused)
// through the runtime's driver entry point, so the library does not link
// against libcuda.  Null when the driver does not provide it.
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetIdFn ctx_get_id() {
  static CtxGetIdFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetIdFn>(ptr);
  });
  return fn;
}

// Device address of the scratch array in the current context.  The lookup is
// made once per context and cached per device with the context's id; when the
// id cannot be read the address is looked up on every call.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_UNSUPPORTED;
  // (no context current yet: the id read fails and the address is looked up,
  // which also makes the device's primary context current)
  unsigned long long id = 0;
  const CtxGetIdFn get_id = ctx_get_id();
  const bool have_id = get_id != nullptr && get_id(nullptr, &id) == CUDA_SUCCESS && id != 0;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (have_id && g_scratch[dev].addr != nullptr && g_scratch[dev].ctx_id == id) {
    *out = g_scratch[dev].addr;
    return PKV_OK;
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) return PKV_ERR_CUDA;
  g_scratch[dev].ctx_id = have_id ? id : 0;
  g_scratch[dev].addr = have_id ? p : nullptr;
  *out = p;
  return PKV_OK;
}

}  // namespace

extern "C" int pkv_paged_attention_decode_noalloc(
    void* out, const void* q, pkv_dtype q_dt, const void* k_cache, const void* v_cache,
    pkv_dtype cache_dt, const float* k_scale, const float* v_scale, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, int num_splits, int* err_flag, pkv_stream_t stream) {
  // The same split plan pkv_paged_attention_decode will make (it bounds the
  // context by the block-table capacity first).
  long long cap = (long long)max_blocks_per_seq * block_size;
  int planned_ctx = max_context_len;
  if (max_blocks_per_seq > 0 && block_size > 0 && (long long)planned_ctx > cap)
    planned_ctx = (int)cap;
  const size_t need = pkv_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                         planned_ctx, cache_dt, num_splits);
  if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != PKV_OK) return rc;
  return pkv_paged_attention_decode(out, q, q_dt, k_cache, v_cache, cache_dt, k_scale, v_scale,
                                    block_tables, max_blocks_per_seq, context_lens,
                                    max_context_len, num_seqs, num_q_heads, num_kv_heads,
                                    head_dim, block_size, num_blocks, softmax_scale, scratch,
                                    (size_t)PKV_NOALLOC_SCRATCH_BYTES, num_splits, err_flag,
                                    stream);
}
