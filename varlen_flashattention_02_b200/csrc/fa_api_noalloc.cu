// fa_api_noalloc.cu -- the forward entry point for callers that cannot
// allocate device memory (declared in include/fa_varlen.h as
// fa_varlen_fwd_noalloc).
//
// Some callers cannot call cudaMalloc: code that runs inside another
// framework's plugin or operator interface and is handed only its input and
// output pointers (allocating behind that framework's memory pool breaks its
// accounting), or latency-critical paths where a device allocation, which
// may synchronise the device, is not allowed. For them the forward's scratch
// (the work-list header, per-sequence offsets and the (sequence, tile) list)
// lives in a file-scope device array owned by the library instead of a
// caller-provided workspace.
//
// Host code cannot use the array's name as a device address (on the host it
// is only a stand-in symbol). The address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call made on
// each device, and cached together with the ID of the CUDA context it was
// found in. A device reset (or any new primary context) reloads the module
// and may move the array; the context then has a new ID, so the next call
// looks the address up again instead of using a stale one.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/fa_varlen.h"

namespace {

constexpr int kMaxDevices = 64;

// Every GPU that loads the library holds this buffer until the process exits.
static __device__ __align__(256) unsigned char g_fwd_scratch[FA_NOALLOC_SCRATCH_BYTES];

struct Cached {
  unsigned long long ctx_id;  // ID of the context the address belongs to (0: none yet)
  void* addr;
};
std::mutex g_mutex;
Cached g_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// ID of the calling thread's current context, or 0 if it cannot be told.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_fwd_scratch on the current device (null on failure).
void* scratch_on_current_device(int dev) {
  std::lock_guard<std::mutex> lock(g_mutex);
  const unsigned long long id = current_context_id();
  if (id != 0 && g_cache[dev].ctx_id == id) return g_cache[dev].addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess) return nullptr;
  // The lookup makes the device's primary context current if it was not.
  g_cache[dev] = Cached{id != 0 ? id : current_context_id(), p};
  return p;
}

}  // namespace

extern "C" fa_status_t fa_varlen_fwd_noalloc(const void* q, const void* k, const void* v,
                                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                              int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                                              int num_heads, int head_dim, float softmax_scale, int causal, void* out,
                                              float* softmax_lse, fa_cuda_stream_t stream) {
  // Size check before any CUDA call: the scratch this call needs must fit.
  const size_t need = fa_varlen_fwd_workspace_size(batch, total_q, num_heads, head_dim);
  if (need == 0) return FA_ERR_INVALID_ARGUMENT;
  if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  void* scratch = scratch_on_current_device(dev);
  if (!scratch) return FA_ERR_CUDA;
  // The work-list preparation of the call rewrites every word of the scratch
  // that the forward reads (status, counters, offsets, list), so nothing has
  // to be cleared here.
  return fa_varlen_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q, max_seqlen_k,
                       num_heads, head_dim, softmax_scale, causal, out, softmax_lse, scratch,
                       FA_NOALLOC_SCRATCH_BYTES, stream);
}
