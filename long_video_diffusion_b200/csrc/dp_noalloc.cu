// dp_window_step_noalloc: the window step for callers that cannot allocate device memory.
//
// The regular dp_window_step needs a caller-provided scratch buffer (kv_work) for the
// window's modulated keys and values.  Some callers have no way to get one: code embedded
// in a host that owns all device memory (a framework's caching allocator, a plugin
// interface that hands over only inputs and outputs), or latency-critical loops where a
// cudaMalloc/cudaFree would synchronize the device.  This entry point takes the same
// arguments minus kv_work and uses a fixed array in the library's own device memory
// instead.  It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "dp.h"
#include "dp_internal.h"

namespace {

// The scratch: file-scope device memory of a fixed size.  Every device that loads this
// library holds these bytes until the process exits.  In host code the array's name is
// only a stand-in symbol, never a device address; the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_step_scratch[DP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// The array's address, per device, valid for the CUDA context it was looked up in.  A
// device reset destroys that context (and the module's copy of the array with it); the
// context that replaces it has a new id, so the address is looked up again.
struct ScratchSlot {
  unsigned long long ctx_id = 0;  // 0: not looked up yet
  void* addr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

template <class F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

// Unique id of the calling thread's current context (0 if there is none yet).
bool current_ctx_id(unsigned long long* id) {
  static PfnCtxGetCurrent get_current = driver_fn<PfnCtxGetCurrent>("cuCtxGetCurrent");
  static PfnCtxGetId get_id = driver_fn<PfnCtxGetId>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  if (ctx == nullptr) return true;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// The device address of the array on the current device.  Set-up, once per device and
// context, with that device current: cudaGetSymbolAddress (which also makes the runtime's
// context current if the thread had none).  Later calls compare the context id only.
dp_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dp::set_error(DP_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return dp::set_error(DP_ERR_UNSUPPORTED, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  unsigned long long id = 0;
  if (!current_ctx_id(&id)) return dp::set_error(DP_ERR_CUDA, "cannot read the current CUDA context");
  ScratchSlot& slot = g_scratch[dev];
  if (id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_step_scratch);
    if (e != cudaSuccess || p == nullptr)
      return dp::set_error(DP_ERR_CUDA, "cudaGetSymbolAddress of the step scratch failed");
    if (!current_ctx_id(&id) || id == 0) return dp::set_error(DP_ERR_CUDA, "no current CUDA context after set-up");
    slot.ctx_id = id;
    slot.addr = p;
  }
  *out = slot.addr;
  return DP_OK;
}

}  // namespace

extern "C" dp_status dp_window_step_noalloc(const void* q, const void* k, const void* v, int64_t n_win,
                                            const dp_blocks* blk, dp_kvcache* cache, const void* residual,
                                            void* out, int32_t n_heads, int32_t head_dim, uint32_t flags,
                                            dp_queue* queue, const void* push_noise, int64_t push_rows, dp_dtype dt,
                                            void* stream) {
  if (n_win <= 0 || n_heads <= 0 || head_dim <= 0)
    return dp::set_error(DP_ERR_INVALID_ARG, "n_win, n_heads and head_dim must be positive");
  // k' and v' of the window, in the feature type (f16 for bf16 windows, fp32 for fp32):
  // 2 * n_win * hidden elements.  Compared by division, so no product can overflow.
  const uint64_t feat_bytes = dt == DP_F32 ? 4u : 2u;
  const uint64_t limit = DP_NOALLOC_SCRATCH_BYTES;
  const uint64_t hidden = static_cast<uint64_t>(n_heads) * static_cast<uint64_t>(head_dim);
  const uint64_t row_bytes = hidden <= limit ? 2u * hidden * feat_bytes : limit + 1;
  if (row_bytes > limit || static_cast<uint64_t>(n_win) > limit / row_bytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "window of %lld rows x %llu channels needs more than the %llu scratch bytes of the fixed array",
             static_cast<long long>(n_win), static_cast<unsigned long long>(hidden),
             static_cast<unsigned long long>(limit));
    return dp::set_error(DP_ERR_CAPACITY, msg);
  }
  void* scratch = nullptr;
  dp_status st = scratch_address(&scratch);
  if (st != DP_OK) return st;
  // The prepass writes every k'/v' element of the window before anything reads it, so
  // nothing left in the array by an earlier call is ever used and nothing needs clearing.
  return dp_window_step(q, k, v, n_win, blk, cache, scratch, residual, out, n_heads, head_dim, flags, queue,
                        push_noise, push_rows, dt, stream);
}
