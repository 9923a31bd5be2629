// adaLN modulation prepass and the advance copy kernel — both HBM-bandwidth bound.
//
// Modulation (each block conditioned on its own timestep: "Minute-Long Videos with Dual
// Parallelisms", abstract, blocks at progressively decreasing noise levels; pith.science
// review, Section 3.1): y = x * (1 + scale_b) + shift_b per channel, one fp32 FMA per
// element, rounded once to the element type.  Each thread moves 16-byte vectors (8 bf16
// or 4 fp32) with four independent vectors in flight; the grid is a multiple of the SM
// count and strides over all rows of every segment.
//
// Copy (the queue advance: the exiting block's K'/V' rows become the cache, a fresh noise
// block enters the latent ring; review, key machinery and Section 3.2): up to four
// (src, dst, bytes) segments in one launch, 16-byte vectors, bit-exact.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dp_internal.h"

namespace dp {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct ModSegs {
  const uint4* src[2];
  uint4* dst[2];
};

__device__ __forceinline__ uint4 mod_vec_bf16(uint4 x, const float* sh, const float* sc) {
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(sh)), s1 = __ldg(reinterpret_cast<const float4*>(sh) + 1);
  const float4 c0 = __ldg(reinterpret_cast<const float4*>(sc)), c1 = __ldg(reinterpret_cast<const float4*>(sc) + 1);
  const float shv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const float scv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(x2[e]);
    __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(f.x, 1.0f + scv[2 * e], shv[2 * e]),
                                             fmaf(f.y, 1.0f + scv[2 * e + 1], shv[2 * e + 1]));
    o[e] = *reinterpret_cast<uint32_t*>(&r);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 mod_vec_f32(uint4 x, const float* sh, const float* sc) {
  const float4 s = __ldg(reinterpret_cast<const float4*>(sh));
  const float4 c = __ldg(reinterpret_cast<const float4*>(sc));
  float4 f = *reinterpret_cast<float4*>(&x);
  f.x = fmaf(f.x, 1.0f + c.x, s.x);
  f.y = fmaf(f.y, 1.0f + c.y, s.y);
  f.z = fmaf(f.z, 1.0f + c.z, s.z);
  f.w = fmaf(f.w, 1.0f + c.w, s.w);
  return *reinterpret_cast<uint4*>(&f);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) modulate_kernel(ModSegs segs, uint32_t vec_per_row, uint32_t vec_per_seg,
                                                            int hidden, BlockTable bt) {
  constexpr int VE = BF16 ? 8 : 4;  // elements per 16-byte vector
  const uint4* src = segs.src[blockIdx.y];
  uint4* dst = segs.dst[blockIdx.y];
  const uint32_t stride = gridDim.x * kThreads;
  for (uint32_t base = blockIdx.x * kThreads + threadIdx.x; base < vec_per_seg; base += stride * kUnroll) {
    uint4 x[kUnroll];
    uint32_t idx[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      idx[u] = base + u * stride;
      if (idx[u] < vec_per_seg) x[u] = __ldcs(src + idx[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (idx[u] >= vec_per_seg) break;
      const uint32_t row = idx[u] / vec_per_row;
      const uint32_t col = (idx[u] - row * vec_per_row) * VE;
      const float* m = block_mod(bt, block_of_row(bt, row));
      const uint4 y = BF16 ? mod_vec_bf16(x[u], m + col, m + hidden + col) : mod_vec_f32(x[u], m + col, m + hidden + col);
      dst[idx[u]] = y;
    }
  }
}

struct CopySegs {
  const uint4* src[kMaxCopySegs];
  uint4* dst[kMaxCopySegs];
  uint32_t n_vec[kMaxCopySegs];
};

__global__ void __launch_bounds__(kThreads) copy_kernel(CopySegs segs) {
  const uint4* src = segs.src[blockIdx.y];
  uint4* dst = segs.dst[blockIdx.y];
  const uint32_t n = segs.n_vec[blockIdx.y];
  const uint32_t stride = gridDim.x * kThreads;
  for (uint32_t base = blockIdx.x * kThreads + threadIdx.x; base < n; base += stride * kUnroll) {
    uint4 x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (base + u * stride < n) x[u] = __ldcs(src + base + u * stride);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (base + u * stride < n) dst[base + u * stride] = x[u];
  }
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

unsigned grid_for(uint64_t n_vec) {
  const uint64_t per_cta = static_cast<uint64_t>(kThreads) * kUnroll;
  const uint64_t want = (n_vec + per_cta - 1) / per_cta;
  const uint64_t cap = static_cast<uint64_t>(sm_count()) * 8;  // 8 resident CTAs of 256 threads per SM
  const uint64_t g = want < cap ? want : cap;
  return static_cast<unsigned>(g > 0 ? g : 1);
}

}  // namespace

cudaError_t launch_modulate(const void* const* src, void* const* dst, int nseg, int64_t n_rows, int hidden,
                            const BlockTable& bt, dp_dtype dt, cudaStream_t s) {
  if (nseg < 1 || nseg > 2 || n_rows <= 0) return cudaErrorInvalidValue;
  const int eb = dt == DP_BF16 ? 2 : 4;
  const uint64_t vpr = static_cast<uint64_t>(hidden) * eb / 16;
  const uint64_t vps = vpr * static_cast<uint64_t>(n_rows);
  if (vps >= (1ull << 31)) return cudaErrorInvalidValue;
  ModSegs segs;
  for (int i = 0; i < 2; ++i) {
    const int j = i < nseg ? i : 0;
    segs.src[i] = static_cast<const uint4*>(src[j]);
    segs.dst[i] = static_cast<uint4*>(dst[j]);
  }
  dim3 grid(grid_for(vps), nseg);
  if (dt == DP_BF16)
    modulate_kernel<true><<<grid, kThreads, 0, s>>>(segs, static_cast<uint32_t>(vpr), static_cast<uint32_t>(vps), hidden, bt);
  else
    modulate_kernel<false><<<grid, kThreads, 0, s>>>(segs, static_cast<uint32_t>(vpr), static_cast<uint32_t>(vps), hidden, bt);
  return cudaGetLastError();
}

cudaError_t launch_copy(const CopySeg* segs, int nseg, cudaStream_t s) {
  CopySegs cs;
  int n = 0;
  uint64_t maxv = 0;
  for (int i = 0; i < nseg; ++i) {
    if (segs[i].bytes <= 0) continue;
    if (segs[i].bytes % 16) return cudaErrorInvalidValue;
    const uint64_t nv = static_cast<uint64_t>(segs[i].bytes) / 16;
    if (nv >= (1ull << 31)) return cudaErrorInvalidValue;
    cs.src[n] = static_cast<const uint4*>(segs[i].src);
    cs.dst[n] = static_cast<uint4*>(segs[i].dst);
    cs.n_vec[n] = static_cast<uint32_t>(nv);
    maxv = nv > maxv ? nv : maxv;
    ++n;
  }
  if (n == 0) return cudaSuccess;
  for (int i = n; i < kMaxCopySegs; ++i) {
    cs.src[i] = nullptr;
    cs.dst[i] = nullptr;
    cs.n_vec[i] = 0;
  }
  dim3 grid(grid_for(maxv), n);
  copy_kernel<<<grid, kThreads, 0, s>>>(cs);
  return cudaGetLastError();
}

}  // namespace dp
