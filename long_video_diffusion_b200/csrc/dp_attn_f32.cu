// Window attention in full fp32 on the CUDA cores (DP_F32 inputs).
//
// Same operation as the tensor-core path ("Minute-Long Videos with Dual Parallelisms",
// abstract; pith.science review, Section 3.2): per head, each window query attends to the
// valid cache rows and then to every window row, with the adaLN modulation of q in the
// prologue and the per-block gate (+ residual) in the epilogue.  fp32 inputs ask for
// agreement to 1e-4, which tf32 tensor cores (10-bit mantissa) cannot give, so this path
// uses FFMA: one thread owns one (query row, head), keys stream through shared memory in
// tiles of 32 rows, and the softmax is online (running max and sum, exp via expf).
#include <cuda_runtime.h>

#include <cmath>

#include "dp_internal.h"

namespace dp {

namespace {

constexpr int kRows = 64;   // query rows (threads) per CTA
constexpr int kKeys = 32;   // keys per shared-memory tile

template <int HD>
__global__ void __launch_bounds__(kRows) attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                                         const float* __restrict__ v, const float* __restrict__ ck,
                                                         const float* __restrict__ cv, const float* __restrict__ res,
                                                         float* __restrict__ out, int64_t n_win, CacheSegs segs,
                                                         int hidden, float scale, uint32_t flags, BlockTable bt) {
  __shared__ float sk[kKeys][HD];
  __shared__ float sv[kKeys][HD];
  const int head = blockIdx.y;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRows + threadIdx.x;
  const bool row_ok = row < n_win;
  const int b = row_ok ? block_of_row(bt, row) : 0;
  const float* modb = block_mod(bt, b);

  float qr[HD];
  float acc[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) {
    float x = row_ok ? q[row * hidden + head * HD + d] : 0.0f;
    if (row_ok && (flags & DP_MOD_Q)) x = fmaf(x, 1.0f + modb[hidden + head * HD + d], modb[head * HD + d]);
    qr[d] = x * scale;
    acc[d] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;

  // the cache segments, then the window
  for (int seg = 0; seg <= segs.n; ++seg) {
    const bool in_cache = seg < segs.n;
    const int64_t base = in_cache ? pick(segs.row, seg) : 0;
    const float* K = in_cache ? ck + base * hidden : k;
    const float* V = in_cache ? cv + base * hidden : v;
    const int64_t len = in_cache ? pick(segs.len, seg) : n_win;
    for (int64_t j0 = 0; j0 < len; j0 += kKeys) {
      const int nk = (len - j0) < kKeys ? static_cast<int>(len - j0) : kKeys;
      __syncthreads();
      for (int e = threadIdx.x; e < kKeys * HD; e += kRows) {
        const int jj = e / HD, d = e % HD;
        const bool in = jj < nk;
        sk[jj][d] = in ? K[(j0 + jj) * hidden + head * HD + d] : 0.0f;
        sv[jj][d] = in ? V[(j0 + jj) * hidden + head * HD + d] : 0.0f;
      }
      __syncthreads();
      for (int jj = 0; jj < nk; ++jj) {
        float s = 0.0f;
#pragma unroll
        for (int d = 0; d < HD; ++d) s = fmaf(qr[d], sk[jj][d], s);
        if (s > m) {
          const float f = expf(m - s);
          l *= f;
#pragma unroll
          for (int d = 0; d < HD; ++d) acc[d] *= f;
          m = s;
        }
        const float pj = expf(s - m);
        l += pj;
#pragma unroll
        for (int d = 0; d < HD; ++d) acc[d] = fmaf(pj, sv[jj][d], acc[d]);
      }
    }
  }
  if (!row_ok) return;
  const float inv = 1.0f / l;
#pragma unroll
  for (int d = 0; d < HD; ++d) {
    const int64_t idx = row * hidden + head * HD + d;
    float o = acc[d] * inv;
    if (flags & DP_GATE_OUT) o *= modb[2 * hidden + head * HD + d];
    if (res) o += res[idx];
    out[idx] = o;
  }
}

template <int HD>
cudaError_t launch_hd(const AttnArgs& a, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((a.n_win + kRows - 1) / kRows), static_cast<unsigned>(a.n_heads));
  attn_f32_kernel<HD><<<grid, kRows, 0, s>>>(
      static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.v),
      static_cast<const float*>(a.cache_k), static_cast<const float*>(a.cache_v), static_cast<const float*>(a.residual),
      static_cast<float*>(a.out), a.n_win, a.segs, a.hidden, a.softmax_scale, a.flags, a.bt);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t s) {
  switch (a.head_dim) {
    case 4: return launch_hd<4>(a, s);
    case 8: return launch_hd<8>(a, s);
    case 16: return launch_hd<16>(a, s);
    case 32: return launch_hd<32>(a, s);
    case 64: return launch_hd<64>(a, s);
    case 128: return launch_hd<128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dp
