// adaLN modulation prepass and the advance copy kernel — both HBM-bandwidth bound.
//
// Modulation (each block conditioned on its own timestep: "Minute-Long Videos with Dual
// Parallelisms", abstract, blocks at progressively decreasing noise levels; pith.science
// review, Section 3.1): y = x * (1 + scale_b) + shift_b per channel, one fp32 FMA per
// element, rounded once to the output type (f16 saturates at +-65504).
//
// Copy (the queue advance: the exiting block's K'/V' rows become the cache, a fresh noise
// block enters the latent ring; review, key machinery and Section 3.2): up to four
// (src, dst, bytes) segments in one launch, 16-byte vectors, bit-exact.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dp_device.cuh"
#include "dp_internal.h"

namespace dp {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;      // 16-byte vectors a copy thread has in flight
constexpr int kGridUnroll = 4;  // the copy grid is sized as if each thread moved 4 (small copies keep their CTAs)

// Element formats of a 16-byte vector: 8 bf16, 8 f16 or 4 fp32.
enum Fmt { kBF16 = 0, kF16 = 1, kF32 = 2 };

template <int F>
__device__ __forceinline__ void unpack8(uint4 x, float (&f)[8]) {
  if constexpr (F == kBF16) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 t = __bfloat1622float2(h[e]);
      f[2 * e] = t.x;
      f[2 * e + 1] = t.y;
    }
  } else if constexpr (F == kF16) {
    const __half2* h = reinterpret_cast<const __half2*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 t = __half22float2(h[e]);
      f[2 * e] = t.x;
      f[2 * e + 1] = t.y;
    }
  } else {
    const float4 t = *reinterpret_cast<const float4*>(&x);
    f[0] = t.x, f[1] = t.y, f[2] = t.z, f[3] = t.w;
  }
}

template <int F>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  if constexpr (F == kBF16) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  } else if constexpr (F == kF16) {
    return make_uint4(pack_f16x2_sat(f[0], f[1]), pack_f16x2_sat(f[2], f[3]), pack_f16x2_sat(f[4], f[5]),
                      pack_f16x2_sat(f[6], f[7]));
  } else {
    const float4 t = make_float4(f[0], f[1], f[2], f[3]);
    return *reinterpret_cast<const uint4*>(&t);
  }
}

// One CTA thread per 16-byte column vector of a row (blockDim = vectors per row, up to
// 1024; wider rows loop); the CTA walks rows kRowsInFlight at a time, grid-striding over the
// rows of its segment (grid.y).  A thread keeps its columns' shift and 1 + scale in
// registers and reloads them only when the row's block changes, so HBM traffic is the 16
// bytes read and written per vector and nothing else.  Two rows in flight: inside the
// window step, at the power-capped SM clock the attention leaves behind, this ran at 0.77 of
// HBM bandwidth on the 131,072-token window against 0.69 with four rows (both 0.84 alone).
constexpr int kRowsInFlight = 2;

template <int FI, int FO>
__global__ void __launch_bounds__(1024) modulate_kernel(const uint4* __restrict__ src0, uint4* __restrict__ dst0,
                                                        const uint4* __restrict__ src1, uint4* __restrict__ dst1,
                                                        uint32_t n_rows, uint32_t vec_per_row, int hidden,
                                                        BlockTable bt) {
  constexpr int VE = FI == kF32 ? 4 : 8;  // elements per 16-byte vector
  const uint4* src = blockIdx.y ? src1 : src0;
  uint4* dst = blockIdx.y ? dst1 : dst0;
  for (uint32_t cv = threadIdx.x; cv < vec_per_row; cv += blockDim.x) {
    const uint32_t col = cv * VE;
    int cur = -1;
    float sh[VE], a[VE];
    for (uint32_t r0 = blockIdx.x * kRowsInFlight; r0 < n_rows; r0 += gridDim.x * kRowsInFlight) {
      uint4 x[kRowsInFlight];
#pragma unroll
      for (int u = 0; u < kRowsInFlight; ++u)
        if (r0 + u < n_rows) x[u] = __ldcs(src + static_cast<size_t>(r0 + u) * vec_per_row + cv);
#pragma unroll
      for (int u = 0; u < kRowsInFlight; ++u) {
        const uint32_t row = r0 + u;
        if (row >= n_rows) break;
        const int b = block_of_row(bt, row);
        if (b != cur) {
          const float* m = block_mod(bt, b);
#pragma unroll
          for (int v = 0; v < VE / 4; ++v) {
            const float4 s4 = __ldg(reinterpret_cast<const float4*>(m + col) + v);
            const float4 c4 = __ldg(reinterpret_cast<const float4*>(m + hidden + col) + v);
            sh[4 * v] = s4.x, sh[4 * v + 1] = s4.y, sh[4 * v + 2] = s4.z, sh[4 * v + 3] = s4.w;
            a[4 * v] = 1.0f + c4.x, a[4 * v + 1] = 1.0f + c4.y, a[4 * v + 2] = 1.0f + c4.z, a[4 * v + 3] = 1.0f + c4.w;
          }
          cur = b;
        }
        float f[8];
        unpack8<FI>(x[u], f);
#pragma unroll
        for (int e = 0; e < VE; ++e) f[e] = fmaf(f[e], a[e], sh[e]);
        dst[static_cast<size_t>(row) * vec_per_row + cv] = pack8<FO>(f);
      }
    }
  }
}

// Pre-norm and modulation of the DiT attention sublayer (adaLN: the block's shift and scale
// applied to the layer-normed hidden state): h = (x - mean) / sqrt(var + eps) * (1 + scale_b)
// + shift_b, mean and var over the row's channels in fp32 (two passes), rounded once to
// bf16.  One warp per row; lane l handles the row's 16-byte vectors l, l + 32, ...  The row
// is read three times (sum, squared deviations, output) rather than held in registers: the
// second and third reads hit L1/L2, and the few registers leave room for 64 warps per SM,
// which is what hides the memory latency of a one-row-per-warp reduction.
constexpr int kLnWarps = 8;

__global__ void __launch_bounds__(32 * kLnWarps) ln_modulate_kernel(const uint4* __restrict__ x, uint4* __restrict__ h,
                                                                   uint32_t n_rows, int hidden, float eps,
                                                                   BlockTable bt) {
  const int lane = threadIdx.x & 31;
  const uint32_t row = blockIdx.x * kLnWarps + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int vpr = hidden / 8;  // 16-byte vectors per row
  const uint4* xr = x + static_cast<size_t>(row) * vpr;
  float sum = 0.0f;
#pragma unroll 4
  for (int i = lane; i < vpr; i += 32) {
    float f[8];
    unpack8<kBF16>(__ldg(xr + i), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) sum += f[e];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / static_cast<float>(hidden);
  float sq = 0.0f;
#pragma unroll 4
  for (int i = lane; i < vpr; i += 32) {
    float f[8];
    unpack8<kBF16>(__ldg(xr + i), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float d = f[e] - mean;
      sq = fmaf(d, d, sq);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = 1.0f / sqrtf(sq / static_cast<float>(hidden) + eps);
  const float* m = block_mod(bt, block_of_row(bt, row));
  uint4* hr = h + static_cast<size_t>(row) * vpr;
#pragma unroll 2
  for (int i = lane; i < vpr; i += 32) {
    const int col = i * 8;
    float f[8];
    unpack8<kBF16>(__ldg(xr + i), f);
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(m + col));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(m + col + 4));
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(m + hidden + col));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(m + hidden + col + 4));
    const float sh[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    const float sc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = fmaf((f[e] - mean) * rstd, 1.0f + sc[e], sh[e]);
    __stcs(hr + i, pack8<kBF16>(f));
  }
}

struct CopySegs {
  const uint4* src[kMaxCopySegs];
  uint4* dst[kMaxCopySegs];
  uint32_t n_vec[kMaxCopySegs];
};

__global__ void __launch_bounds__(kThreads) copy_kernel(CopySegs segs) {
  // segment selected with constant indices (no run-time indexing of the kernel argument)
  const uint32_t y = blockIdx.y;
  const uint4* src = segs.src[0];
  uint4* dst = segs.dst[0];
  uint32_t n = segs.n_vec[0];
#pragma unroll
  for (int i = 1; i < kMaxCopySegs; ++i)
    if (y == static_cast<uint32_t>(i)) {
      src = segs.src[i];
      dst = segs.dst[i];
      n = segs.n_vec[i];
    }
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

// Gather of whole latent frames from a noise pool into a queue slot and its mirror (the
// coordinated noise initialisation's push: each new block is a shuffled selection of the
// pool's frames).  grid.y = output frame; byte copy, bit-exact.
__global__ void __launch_bounds__(kThreads) gather_frames_kernel(FrameGather g) {
  const int f = blockIdx.y;
  const uint4* src = g.pool + static_cast<size_t>(pick(g.idx, f)) * g.vec_per_frame;
  uint4* d0 = g.dst0 + static_cast<size_t>(f) * g.vec_per_frame;
  uint4* d1 = g.dst1 + static_cast<size_t>(f) * g.vec_per_frame;
  const uint32_t stride = gridDim.x * kThreads;
  for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < g.vec_per_frame; i += stride) {
    const uint4 v = __ldcs(src + i);
    d0[i] = v;
    d1[i] = v;
  }
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

unsigned grid_for(uint64_t n_vec) {
  const uint64_t per_cta = static_cast<uint64_t>(kThreads) * kGridUnroll;
  const uint64_t want = (n_vec + per_cta - 1) / per_cta;
  const uint64_t cap = static_cast<uint64_t>(sm_count()) * 8;  // 8 resident CTAs of 256 threads per SM
  const uint64_t g = want < cap ? want : cap;
  return static_cast<unsigned>(g > 0 ? g : 1);
}

}  // namespace

cudaError_t launch_modulate(const void* const* src, void* const* dst, int nseg, int64_t n_rows, int hidden,
                            const BlockTable& bt, dp_dtype x_dt, dp_dtype y_dt, cudaStream_t s) {
  if (nseg < 1 || nseg > 2 || n_rows <= 0 || n_rows >= (1ll << 31)) return cudaErrorInvalidValue;
  const int eb = x_dt == DP_F32 ? 4 : 2;
  const uint32_t vpr = static_cast<uint32_t>(static_cast<int64_t>(hidden) * eb / 16);
  const unsigned threads = vpr >= 1024 ? 1024u : ((vpr + 31u) / 32u) * 32u;
  // enough CTAs to fill every SM several times over, each with its own rows
  const uint64_t row_groups = (static_cast<uint64_t>(n_rows) + kRowsInFlight - 1) / kRowsInFlight;
  const uint64_t per_sm = 2048 / threads > 0 ? 2048 / threads : 1;
  const uint64_t cap = static_cast<uint64_t>(sm_count()) * per_sm * 2;
  dim3 grid(static_cast<unsigned>(row_groups < cap ? row_groups : cap), nseg);
  const uint4* s0 = static_cast<const uint4*>(src[0]);
  uint4* d0 = static_cast<uint4*>(dst[0]);
  const uint4* s1 = static_cast<const uint4*>(src[nseg > 1 ? 1 : 0]);
  uint4* d1 = static_cast<uint4*>(dst[nseg > 1 ? 1 : 0]);
  const uint32_t nr = static_cast<uint32_t>(n_rows);
  if (x_dt == DP_BF16 && y_dt == DP_BF16)
    modulate_kernel<kBF16, kBF16><<<grid, threads, 0, s>>>(s0, d0, s1, d1, nr, vpr, hidden, bt);
  else if (x_dt == DP_BF16 && y_dt == DP_F16)
    modulate_kernel<kBF16, kF16><<<grid, threads, 0, s>>>(s0, d0, s1, d1, nr, vpr, hidden, bt);
  else if (x_dt == DP_F16 && y_dt == DP_F16)
    modulate_kernel<kF16, kF16><<<grid, threads, 0, s>>>(s0, d0, s1, d1, nr, vpr, hidden, bt);
  else if (x_dt == DP_F32 && y_dt == DP_F32)
    modulate_kernel<kF32, kF32><<<grid, threads, 0, s>>>(s0, d0, s1, d1, nr, vpr, hidden, bt);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_ln_modulate(const void* x, void* h, int64_t n_rows, int hidden, float eps, const BlockTable& bt,
                               cudaStream_t s) {
  if (n_rows <= 0 || n_rows >= (1ll << 31) || hidden % 256 || hidden > 8192) return cudaErrorInvalidValue;
  const uint64_t grid = (static_cast<uint64_t>(n_rows) + kLnWarps - 1) / kLnWarps;
  ln_modulate_kernel<<<static_cast<unsigned>(grid), 32 * kLnWarps, 0, s>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(h), static_cast<uint32_t>(n_rows), hidden, eps, bt);
  return cudaGetLastError();
}

cudaError_t launch_gather_frames(const FrameGather& g, cudaStream_t s) {
  if (g.n_frames < 1 || g.n_frames > kMaxGatherFrames || g.vec_per_frame == 0) return cudaErrorInvalidValue;
  const uint64_t per_frame =
      (static_cast<uint64_t>(g.vec_per_frame) + kThreads * kGridUnroll - 1) / (kThreads * kGridUnroll);
  const uint64_t cap = (static_cast<uint64_t>(sm_count()) * 8 + g.n_frames - 1) / g.n_frames;
  dim3 grid(static_cast<unsigned>(per_frame < cap ? (per_frame > 0 ? per_frame : 1) : cap),
            static_cast<unsigned>(g.n_frames));
  gather_frames_kernel<<<grid, kThreads, 0, s>>>(g);
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
