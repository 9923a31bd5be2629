// Linear layers of the DiT attention sublayer on the sm_100a tensor cores: y = a W^T + bias.
//
// The pages' DiT (the review's Section 3.2: each block's tokens pass through the model's
// self-attention, whose K/V features the cache keeps) projects the pre-normed, modulated
// hidden states h to q, k, v and projects the attention output back with a gated residual
// (DiT adaLN: x + gate_b * (o W_o^T + b_o)).  Trained weights are out of reach here; the
// kernels run on synthetic weights with the real shapes.
//
//   a: [m][k] bf16 row-major (K contiguous), W: [n][k] bf16 (out-features x in-features,
//   K contiguous), fp32 accumulation in tensor memory.
//
// Design (one CTA = one 128 x BN output tile, BN = 256 or 128):
//   warp 0     TMA producer: the A tile (128 x 64) and the W tile (BN x 64) of each K step
//              (64 bf16 = one 128-byte swizzle row) into a ring of shared-memory stages
//   warp 1     MMA issuer: four 128 x BN x 16 tcgen05.mma per K step, accumulator in BN
//              tensor-memory columns; owns the tensor memory
//   warps 2-5  epilogue: one thread per output row (TMEM lane), 32 columns at a time:
//              bias, then the variant's store (plain, q/k/v split, gated residual)
// CTAs walk the n tiles of one m tile consecutively, so W (at most 57 MB here) stays in L2
// while the A row block is reused from L2 across the n tiles.
// Every wait is bounded (dp_device.cuh): on giving up the kernel records a timeout in the
// device status word, stops, drains its own copies and products, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dp_device.cuh"
#include "dp_internal.h"

namespace dp {

namespace {

constexpr int GBM = 128;  // output rows per tile
constexpr int GBK = 64;   // K per stage: one 128-byte swizzle row of bf16

template <int BN>
struct GemmLayout {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = GBM * GBK * 2;
  static constexpr int B_BYTES = BN * GBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // full[S], empty[S], acc, fin
  static constexpr int N_BAR = 2 * STAGES + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1 KB
  static constexpr int kThreads = 192;
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(BN == 128 || BN == 256, "tile width");
};

struct GemmParams {
  int64_t m;
  int32_t n;
  int32_t k;
  int32_t n_tiles_n;
  const float* bias;               // [n] or NULL
  void* y0;                        // kEpiStore: y; kEpiQKV: q; kEpiGateResidual: y
  void* y1;                        // kEpiQKV: k
  void* y2;                        // kEpiQKV: v
  int32_t ld_y;                    // row pitch of the outputs, elements
  int32_t seg_cols;                // kEpiQKV: columns per q/k/v segment (hidden)
  int32_t y_f16;                   // kEpiStore: output f16 (1) or bf16 (0)
  const __nv_bfloat16* residual;   // kEpiGateResidual: [m][n]
  uint32_t* status;
  BlockTable bt;                   // kEpiGateResidual: gate of the row's block
};

template <int EPI>
__device__ __forceinline__ void store32(const GemmParams& p, int64_t row, int col, const float (&v)[32]) {
  // v: 32 consecutive output columns col .. col + 31 of `row`, bias already added
  if constexpr (EPI == kEpiStore) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y0) + row * p.ld_y + col);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float* f = v + 8 * c;
      dst[c] = p.y_f16 ? make_uint4(pack_f16x2_sat(f[0], f[1]), pack_f16x2_sat(f[2], f[3]),
                                    pack_f16x2_sat(f[4], f[5]), pack_f16x2_sat(f[6], f[7]))
                       : make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                    pack_bf16x2(f[6], f[7]));
    }
  } else if constexpr (EPI == kEpiQKV) {
    // q (bf16, the attention's raw query) | k | v (f16 features, saturating)
    const int seg = col / p.seg_cols;
    const int cin = col - seg * p.seg_cols;
    void* base = seg == 0 ? p.y0 : (seg == 1 ? p.y1 : p.y2);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(base) + row * p.ld_y + cin);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float* f = v + 8 * c;
      dst[c] = seg == 0 ? make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                     pack_bf16x2(f[6], f[7]))
                        : make_uint4(pack_f16x2_sat(f[0], f[1]), pack_f16x2_sat(f[2], f[3]),
                                     pack_f16x2_sat(f[4], f[5]), pack_f16x2_sat(f[6], f[7]));
    }
  } else {
    // y = residual + gate_b * (a W^T + bias), b = block of the row
    const float* gate = block_mod(p.bt, block_of_row(p.bt, row)) + 2 * static_cast<int64_t>(p.n) + col;
    const uint4* res = reinterpret_cast<const uint4*>(p.residual + row * p.n + col);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.y0) + row * p.ld_y + col);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 r = res[c];
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&r);
      const float4 g0 = *reinterpret_cast<const float4*>(gate + 8 * c);
      const float4 g1 = *reinterpret_cast<const float4*>(gate + 8 * c + 4);
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float o[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 rf = __bfloat1622float2(r2[e]);
        o[2 * e] = fmaf(g[2 * e], v[8 * c + 2 * e], rf.x);
        o[2 * e + 1] = fmaf(g[2 * e + 1], v[8 * c + 2 * e + 1], rf.y);
      }
      dst[c] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                          pack_bf16x2(o[6], o[7]));
    }
  }
}

// Bounded wait that ignores the abort flag: used to drain work this CTA already issued.
__device__ __forceinline__ void gemm_drain_wait(uint32_t bar, uint32_t parity, uint32_t* status) {
  const long long t0 = sm_clock();
  while (!mbar_try_wait(bar, parity)) {
    if (sm_clock() - t0 > kWaitLimitCycles) {
      atomicOr(status, DEV_ERR_TIMEOUT_DRAIN);
      return;
    }
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(GemmLayout<BN>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const GemmParams p) {
  using L = GemmLayout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x / p.n_tiles_n;  // consecutive CTAs share the A row block
  const int n_tile = blockIdx.x % p.n_tiles_n;
  const int KT = (p.k + GBK - 1) / GBK;

  const uint32_t bar0 = sb + L::OFF_BAR;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (L::STAGES + s); };
  const uint32_t acc = bar0 + 8u * (2 * L::STAGES);
  const uint32_t fin = bar0 + 8u * (2 * L::STAGES + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(acc, 1);
    mbar_init(fin, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), BN);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % L::STAGES;
        if (kt >= L::STAGES &&
            !mbar_wait(empty(s), ((kt / L::STAGES) - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_EMPTY))
          break;
        const uint32_t st = sb + s * L::STAGE_BYTES;
        mbar_arrive_expect_tx(full(s), L::STAGE_BYTES);
        tma_load_2d(st, &tm_a, kt * GBK, m_tile * GBM, full(s));
        tma_load_2d(st + L::A_BYTES, &tm_b, kt * GBK, n_tile * BN, full(s));
        issued = kt + 1;
      }
      // every copy this CTA issued lands before its shared memory is released
      const int first = issued > L::STAGES ? issued - L::STAGES : 0;
      for (int kt = first; kt < issued; ++kt) gemm_drain_wait(full(kt % L::STAGES), (kt / L::STAGES) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1u /* bf16 */, GBM, BN, false);
      const uint64_t da0 = sdesc_sw128(sb, 16, 1024);
      const uint64_t db0 = sdesc_sw128(sb + L::A_BYTES, 16, 1024);
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % L::STAGES;
        ok = mbar_wait(full(s), (kt / L::STAGES) & 1, abort, p.status, DEV_ERR_TIMEOUT_KV);
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = static_cast<uint64_t>((s * L::STAGE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < GBK / 16; ++kk)
          mma_ss(tmem, da0 + so + kk * 2, db0 + so + kk * 2, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(empty(s));  // the stage is free once these products have read it
      }
      if (ok) mma_commit(acc);
      // every product issued completes before TMEM is released
      mma_commit(fin);
      gemm_drain_wait(fin, 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    bool ok = mbar_wait(acc, 0, abort, p.status, DEV_ERR_TIMEOUT_O);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int quarter = warp & 3;  // TMEM lanes this warp may access
      const int64_t row = static_cast<int64_t>(m_tile) * GBM + quarter * 32 + lane;
      const uint32_t taddr = tmem + ((static_cast<uint32_t>(quarter) * 32u) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        const int col = n_tile * BN + c0;
        if (col >= p.n) break;  // uniform across the CTA
        uint32_t r[32];
        tmem_ld32(taddr + c0, r);
        tmem_wait_ld();
        if (row < p.m) {
          float v[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = __uint_as_float(r[c]);
          if (p.bias) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 b = *reinterpret_cast<const float4*>(p.bias + col + c);
              v[c] += b.x;
              v[c + 1] += b.y;
              v[c + 2] += b.z;
              v[c + 3] += b.w;
            }
          }
          store32<EPI>(p, row, col, v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

template <int BN, int EPI>
cudaError_t launch_bn(const GemmArgs& g, cudaStream_t s) {
  using L = GemmLayout<BN>;
  CUtensorMap ta, tb;
  if (!encode_tmap_16(&ta, g.a, g.m, g.k, GBM, false) || !encode_tmap_16(&tb, g.w, g.n, g.k, BN, false))
    return cudaErrorInvalidValue;
  GemmParams p;
  p.m = g.m;
  p.n = g.n;
  p.k = g.k;
  p.n_tiles_n = (g.n + BN - 1) / BN;
  p.bias = g.bias;
  p.y0 = g.y0;
  p.y1 = g.y1;
  p.y2 = g.y2;
  p.ld_y = g.ld_y;
  p.seg_cols = g.seg_cols;
  p.y_f16 = g.y_f16;
  p.residual = static_cast<const __nv_bfloat16*>(g.residual);
  p.status = g.status;
  p.bt = g.bt;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};  // per instantiation and device
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t m_tiles = (g.m + GBM - 1) / GBM;
  const int64_t grid = m_tiles * p.n_tiles_n;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  gemm_tc_kernel<BN, EPI><<<static_cast<unsigned>(grid), L::kThreads, L::ALLOC, s>>>(ta, tb, p);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_epi(const GemmArgs& g, cudaStream_t s) {
  // the widest tile that divides the columns (and, for q/k/v, each segment)
  const int32_t unit = EPI == kEpiQKV ? g.seg_cols : g.n;
  if (unit % 256 == 0) return launch_bn<256, EPI>(g, s);
  return launch_bn<128, EPI>(g, s);
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
  if (g.m <= 0 || g.n <= 0 || g.k <= 0 || g.n % 128 || g.k % 8) return cudaErrorInvalidValue;
  switch (g.epi) {
    case kEpiStore: return launch_epi<kEpiStore>(g, s);
    case kEpiQKV: return launch_epi<kEpiQKV>(g, s);
    case kEpiGateResidual: return launch_epi<kEpiGateResidual>(g, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dp
