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
// Design: a persistent kernel, one CTA per SM, each walking output tiles of 128 x BN (BN =
// 256 or 128) in the order tile = blockIdx.x, blockIdx.x + gridDim.x, ...:
//   warp 0     TMA producer: the A tile (128 x 64) and the W tile (BN x 64) of each K step
//              (64 bf16 = one 128-byte swizzle row) into a ring of shared-memory stages that
//              runs on across tiles
//   warp 1     MMA issuer: four 128 x BN x 16 tcgen05.mma per K step into one of two
//              tensor-memory accumulators (2 x BN columns), alternating per tile; owns the
//              tensor memory
//   warps 2-9  epilogue: two warps per 32-lane quarter of the accumulator, each taking half
//              of the tile's columns; one thread per output row (TMEM lane), 32 columns at a
//              time: bias, then the variant's store (plain, q/k/v split, gated residual,
//              whose residual loads run one chunk ahead); it frees the accumulator for the
//              tile after next, so a tile's epilogue runs while the next tile's products
//              accumulate
// Tiles are numbered in groups of group_m m tiles: within a group the m tiles of one n tile
// are consecutive, so the ~148 tiles in flight span the group's row blocks of A and a few
// column blocks of W.  A group's rows of A stay in L2 while the group sweeps all of W.  A W
// that fits in L2 with room to spare (up to kSmallWBytes) stays there across groups, and
// groups of 16 row blocks keep the rows of A (and of the residual) in flight small; a larger
// W is read from DRAM once per group, so the host then makes the groups as large as about
// kGroupABytes of A allows (equal in size), which reads W a couple of times instead of once
// per 16 row blocks.
// Every wait is bounded (dp_device.cuh): on giving up the kernel records a timeout in the
// device status word, stops, drains its own copies and products, frees TMEM and returns.
#include <atomic>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dp_device.cuh"
#include "dp_internal.h"

namespace dp {

namespace {

constexpr int GBM = 128;  // output rows per tile
constexpr int GBK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int kGroupMSmall = 16;               // m tiles per group while W stays in L2
constexpr int64_t kSmallWBytes = 24ll << 20;   // W up to this size stays in L2 across groups
constexpr int64_t kGroupABytes = 34ll << 20;   // rows of A a group covers when W does not

// Tile t of the grouped order -> (m tile, n tile).
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles_n, int group_m, int& m_tile,
                                            int& n_tile) {
  const int per_group = group_m * n_tiles_n;
  const int group = t / per_group;
  const int first_m = group * group_m;
  const int gm = min(group_m, m_tiles - first_m);
  const int within = t - group * per_group;
  m_tile = first_m + within % gm;
  n_tile = within / gm;
}

template <int BN>
struct GemmLayout {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = GBM * GBK * 2;
  static constexpr int B_BYTES = BN * GBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // full[S], empty[S], acc_full[2], acc_empty[2], fin
  static constexpr int N_BAR = 2 * STAGES + 5;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1 KB
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 32 * (2 + kEpiWarps);
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(BN == 128 || BN == 256, "tile width");
};

struct GemmParams {
  int64_t m;
  int32_t n;
  int32_t k;
  int32_t n_tiles_n;
  int32_t group_m;  // m tiles per group of the tile order
  int32_t m_tiles;
  int32_t n_tiles;
  const float* bias;               // [n] or NULL
  void* y0;                        // kEpiStore: y; kEpiQKV: q; kEpiGateResidual: y
  void* y1;                        // kEpiQKV, kEpiKV: k
  void* y2;                        // kEpiQKV, kEpiKV: v
  int32_t ld_y;                    // row pitch of the outputs, elements
  int32_t seg_cols;                // kEpiQKV, kEpiKV: columns per q/k/v segment (hidden)
  int32_t y_f16;                   // kEpiStore: output f16 (1) or bf16 (0)
  const __nv_bfloat16* residual;   // kEpiGateResidual: [m][n]
  uint32_t* status;
  BlockTable bt;                   // kEpiGateResidual: gate of the row's block
};

// The residual of 32 columns of `row` (kEpiGateResidual), as four 16-byte vectors.
__device__ __forceinline__ void load_res4(const GemmParams& p, int64_t row, int col, uint4 (&r)[4]) {
  const uint4* src = reinterpret_cast<const uint4*>(p.residual + row * p.n + col);
#pragma unroll
  for (int c = 0; c < 4; ++c) r[c] = src[c];
}

template <int EPI>
__device__ __forceinline__ void store32(const GemmParams& p, int64_t row, int col, const float (&v)[32],
                                        const uint4 (&res)[4]) {
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
  } else if constexpr (EPI == kEpiQKV || EPI == kEpiKV) {
    // q (bf16, the attention's raw query) | k | v (f16 features, saturating); kEpiKV has
    // no q columns
    const int sc = col / p.seg_cols;
    const int cin = col - sc * p.seg_cols;
    const int seg = (EPI == kEpiKV ? 1 : 0) + sc;
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
  const int KT = (p.k + GBK - 1) / GBK;
  // this CTA's tiles: blockIdx.x + i * gridDim.x, i < n_mine
  const int n_mine = p.n_tiles > static_cast<int>(blockIdx.x)
                         ? (p.n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / gridDim.x
                         : 0;

  const uint32_t bar0 = sb + L::OFF_BAR;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (L::STAGES + s); };
  auto acc_full = [&](int b) { return bar0 + 8u * (2 * L::STAGES + b); };
  auto acc_empty = [&](int b) { return bar0 + 8u * (2 * L::STAGES + 2 + b); };
  const uint32_t fin = bar0 + 8u * (2 * L::STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 32 * L::kEpiWarps);  // every epilogue thread, after reading the accumulator
    }
    mbar_init(fin, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
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
      int issued = 0;  // K steps issued over all of this CTA's tiles (the ring's position)
      bool ok = true;
      for (int i = 0; ok && i < n_mine; ++i) {
        int m_tile, n_tile;
        tile_coords(blockIdx.x + i * gridDim.x, p.m_tiles, p.n_tiles_n, p.group_m, m_tile, n_tile);
        for (int kt = 0; kt < KT; ++kt) {
          const int g = issued;
          const int s = g % L::STAGES;
          if (g >= L::STAGES &&
              !mbar_wait(empty(s), ((g / L::STAGES) - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t st = sb + s * L::STAGE_BYTES;
          mbar_arrive_expect_tx(full(s), L::STAGE_BYTES);
          tma_load_2d(st, &tm_a, kt * GBK, m_tile * GBM, full(s));
          tma_load_2d(st + L::A_BYTES, &tm_b, kt * GBK, n_tile * BN, full(s));
          issued = g + 1;
        }
      }
      // every copy this CTA issued lands before its shared memory is released
      const int first = issued > L::STAGES ? issued - L::STAGES : 0;
      for (int g = first; g < issued; ++g) mbar_drain_wait(full(g % L::STAGES), (g / L::STAGES) & 1, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(1u /* bf16 */, GBM, BN, false);
      const uint64_t da0 = sdesc_sw128(sb, 16, 1024);
      const uint64_t db0 = sdesc_sw128(sb + L::A_BYTES, 16, 1024);
      bool ok = true;
      int g = 0;  // K steps consumed (the ring's position)
      for (int i = 0; ok && i < n_mine; ++i) {
        const int b = i & 1;
        // the epilogue has read this accumulator's previous tile (i - 2)
        if (i >= 2 && !mbar_wait(acc_empty(b), ((i >> 1) - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_O)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(b * BN);
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int s = g % L::STAGES;
          ok = mbar_wait(full(s), (g / L::STAGES) & 1, abort, p.status, DEV_ERR_TIMEOUT_KV);
          if (!ok) break;
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((s * L::STAGE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < GBK / 16; ++kk)
            mma_ss(d, da0 + so + kk * 2, db0 + so + kk * 2, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
          mma_commit(empty(s));  // the stage is free once these products have read it
        }
        if (ok) mma_commit(acc_full(b));
      }
      // every product issued completes before TMEM is released
      mma_commit(fin);
      mbar_drain_wait(fin, 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9)
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;  // which half of the tile's columns
    constexpr int kCols = BN / 2;
    const uint32_t tlane = (static_cast<uint32_t>(quarter) * 32u) << 16;
    for (int i = 0; i < n_mine; ++i) {
      const int b = i & 1;
      bool ok = mbar_wait(acc_full(b), (i >> 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_O);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      int m_tile, n_tile;
      tile_coords(blockIdx.x + i * gridDim.x, p.m_tiles, p.n_tiles_n, p.group_m, m_tile, n_tile);
      const int64_t row = static_cast<int64_t>(m_tile) * GBM + quarter * 32 + lane;
      const uint32_t taddr = tmem + tlane + static_cast<uint32_t>(b * BN);
      const bool row_ok = row < p.m;
      uint4 res_next[4];  // kEpiGateResidual: the next chunk's residual, loaded one chunk ahead
      if constexpr (EPI == kEpiGateResidual) {
        if (row_ok) load_res4(p, row, n_tile * BN + half * kCols, res_next);
      }
#pragma unroll 1
      for (int c0 = half * kCols; c0 < (half + 1) * kCols; c0 += 32) {
        const int col = n_tile * BN + c0;
        uint4 res[4];
        if constexpr (EPI == kEpiGateResidual) {
#pragma unroll
          for (int c = 0; c < 4; ++c) res[c] = res_next[c];
          if (row_ok && c0 + 32 < (half + 1) * kCols) load_res4(p, row, col + 32, res_next);
        }
        uint32_t r[32];
        tmem_ld32(taddr + c0, r);
        tmem_wait_ld();
        if (row_ok && col < p.n) {
          float v[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = __uint_as_float(r[c]);
          if (p.bias) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 bb = *reinterpret_cast<const float4*>(p.bias + col + c);
              v[c] += bb.x;
              v[c + 1] += bb.y;
              v[c + 2] += bb.z;
              v[c + 3] += bb.w;
            }
          }
          store32<EPI>(p, row, col, v, res);
        }
      }
      // this thread has read its rows of the accumulator: the MMA may reuse it
      tc_fence_before();
      mbar_arrive(acc_empty(b));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
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
  const int64_t m_tiles = (g.m + GBM - 1) / GBM;
  const int64_t n_tiles = m_tiles * p.n_tiles_n;
  if (n_tiles > 0x7fffffff) return cudaErrorInvalidValue;
  p.m_tiles = static_cast<int32_t>(m_tiles);
  p.n_tiles = static_cast<int32_t>(n_tiles);
  if (static_cast<int64_t>(g.n) * g.k * 2 <= kSmallWBytes) {
    p.group_m = kGroupMSmall;
  } else {
    // as few groups as keep a group's rows of A within kGroupABytes, all of about one size
    const int64_t a_tile_bytes = static_cast<int64_t>(GBM) * g.k * 2;
    int64_t groups = (m_tiles * a_tile_bytes + kGroupABytes - 1) / kGroupABytes;
    groups = groups < 1 ? 1 : (groups > m_tiles ? m_tiles : groups);
    p.group_m = static_cast<int32_t>((m_tiles + groups - 1) / groups);
  }
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
  static std::atomic<bool> attr_set[64];  // per instantiation and device (concurrent first calls both set it)
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  int sms = 148;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t grid = n_tiles < sms ? n_tiles : sms;  // one resident CTA per SM, each walking tiles
  gemm_tc_kernel<BN, EPI><<<static_cast<unsigned>(grid), L::kThreads, L::ALLOC, s>>>(ta, tb, p);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_epi(const GemmArgs& g, cudaStream_t s) {
  // the widest tile that divides the columns (and, for q/k/v, each segment)
  const int32_t unit = (EPI == kEpiQKV || EPI == kEpiKV) ? g.seg_cols : g.n;
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
    case kEpiKV: return launch_epi<kEpiKV>(g, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dp
