// dp_window_step_noalloc: the window step for callers that cannot allocate device memory.
//
// The regular dp_window_step needs a caller-provided scratch buffer (kv_work) for the
// window's modulated keys and values.  Some callers have no way to get one: code embedded
// in a host that owns all device memory (a framework's caching allocator, a plugin
// interface that hands over only inputs and outputs), or latency-critical loops where a
// cudaMalloc/cudaFree would synchronize the device.  This entry point takes the same
// arguments minus kv_work and uses a fixed array in the library's own device memory
// instead.  It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
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
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Set-up, once per device, with that device current: the device address of the array.
dp_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dp::set_error(DP_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return dp::set_error(DP_ERR_UNSUPPORTED, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_step_scratch);
    if (e != cudaSuccess || p == nullptr)
      return dp::set_error(DP_ERR_CUDA, "cudaGetSymbolAddress of the step scratch failed");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
  // k' and v' of the window, in the feature type (f16 for bf16 windows, fp32 for fp32)
  const uint64_t feat_bytes = dt == DP_F32 ? 4u : 2u;
  const uint64_t need = 2ull * static_cast<uint64_t>(n_win) * static_cast<uint64_t>(n_heads) *
                        static_cast<uint64_t>(head_dim) * feat_bytes;
  if (need > DP_NOALLOC_SCRATCH_BYTES) {
    char msg[160];
    snprintf(msg, sizeof(msg), "window needs %llu scratch bytes; the fixed scratch holds %llu",
             static_cast<unsigned long long>(need), static_cast<unsigned long long>(DP_NOALLOC_SCRATCH_BYTES));
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
