// Window attention over [cached K/V ; window K/V] on the sm_100a tensor cores.
//
// Operation ("Minute-Long Videos with Dual Parallelisms", abstract: the feature cache of
// the prior block is reused as context; pith.science review, Section 3.2: self-attention
// over the cached K/V of the neighbouring block plus the block's own K/V):
//   q'_i = q_i * (1 + scale_b) + shift_b            (prologue, b = block of row i)
//   o_i  = softmax_j(q'_i . K_j * scale) V_j         (j: cache rows, then window rows)
//   out_i = gate_b * o_i (+ residual_i)              (epilogue)
//
// Operands: the raw window q is bf16; the modulated features q', k', v' and the softmax
// weights P enter the tensor cores as 16-bit values of one type, f16 by default (11-bit
// significand: rounding the modulated features to bf16 alone costs about 2.5e-2 absolute on
// peaked softmaxes, f16 about 3e-3) or bf16; both accumulate in fp32.
//
// Design (one CTA = two 128-row query tiles of one head; keys in tiles of BN rows, 128 at
// head_dim 64 and 64 at head_dim 128):
//   warps 0-3  softmax warpgroup for query tile 0 (one thread per query row)
//   warps 4-7  softmax warpgroup for query tile 1
//   warp 8     TMA producer: K and V tiles into a ring of shared-memory stages
//   warps 9-11 issue the products S_g = Q_g K^T and O_g += P_g V, split so that each warp
//              issues the same number per key tile (head_dim 64: warp 9 S for both query
//              tiles, warps 10-11 PV per tile; head_dim 128: warps 9-10 S per tile, warp 11
//              PV for both); warp 9 also owns the tensor memory
// Registers: launched at kLaunchRegs per thread; the producer/issuer warpgroup gives
// registers back (kLowRegs) and the two softmax warpgroups take them (kHighRegs), so a
// softmax thread can hold its scores without spilling.
// Tensor memory (512 columns): S0, S1 (BN fp32 columns each), O0, O1 (HD columns each) and
// P0, P1 (BN/2 columns each); with these tile widths P always has columns of its own, so the
// next S product runs while the softmax still works on the current tile.  P (16-bit pairs)
// is consumed from TMEM as the A operand of O += P V.  S = Q K^T uses Q and K tiles from shared memory, both K-major with
// the 128-byte swizzle; V is the MN-major B operand of the PV product.
// Softmax is fp32 with exp2 on the MUFU unit (part of it on the FMA pipe,
// see PolyPairs); the running max is only moved (and O
// rescaled) when it grows by more than 2^8, which keeps the result exact because the
// final 1/l uses the same reference max as the numerator.
// The cache part of the keys is one contiguous range of rows (the usual case: the block that
// left) or, in the MULTI instantiation, up to DP_MAX_SLOTS segments of a cache ring (the
// last exited blocks, read together); the single-range code is kept apart because the
// softmax loop's instruction schedule is sensitive to any added per-tile work.
// Every wait is bounded (see dp_device.cuh): on giving up the kernel records a timeout in
// the device status word, stops issuing work, drains its own copies and MMAs, frees TMEM
// and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "dp_device.cuh"
#include "dp_internal.h"

namespace dp {

namespace {

constexpr int BM = 128;          // query rows per tile
constexpr int kTmemCols = 512;
constexpr int kRegFile = 65536;  // 32-bit registers per SM
constexpr float kRescaleLog2 = 8.0f;  // lazy rescale threshold (log2 units)

// exp2 on the FMA pipe for part of the softmax (the MUFU unit retires 16 exp2 per clock per
// SM, no more than the tensor cores need at either head dim): 2^x = 2^n p(f), n = round(x) (added to the
// exponent field), f = x - n in [-1/2, 1/2], p the degree-3 minimax polynomial of 2^f
// (max relative error 7.5e-5, below f16's half ulp), coefficients from
// csrc/fit_exp2_poly.py.  x >= -125 keeps the exponent field positive.
constexpr float kPolyC0 = 0.9999280571937561f;
constexpr float kPolyC1 = 0.6932609677314758f;
constexpr float kPolyC2 = 0.2426111251115799f;
constexpr float kPolyC3 = 0.0551716685295105f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer
constexpr float kPolyMinX = -125.0f;
// Column pairs (of the 16 in each 32-column chunk) whose exponentials use the polynomial: 4
// of 16, spread over the chunk (measured best among 0, 3, 4, 5, 6, 8, 10 and 12 of 16; more
// moves the limit to the issue slots and the FMA pipe, where the polynomial costs about
// seven instructions a pair against one MUFU instruction per exponential).  Where they sit
// changes the compiler's interleaving of the two kinds: at head_dim 64, pairs 0, 5, 10, 15
// ran 3-4 % faster than 0, 4, 8, 12 and than the earlier 6 of 16 (1, 4, 6, 9, 11, 14).
template <int HD>
struct PolyPairs {
  static constexpr uint32_t kMask = HD == 64 ? 0x8421u : 0x1111u;
};

template <int HD>
struct Layout {
  // Query tiles per CTA (one softmax warpgroup each) and keys per tile.  Tensor memory holds
  // S_g (BN fp32 columns), P_g (BN/2 columns of 16-bit pairs) and O_g (HD columns) for each
  // query tile: 128-key tiles at head_dim 64 (448 columns), 64-key tiles at head_dim 128
  // (448 columns; 128-key tiles would leave no room for P, and each query tile would then
  // run S -> softmax -> PV -> S strictly in series).  P therefore always has columns of its
  // own, so the next S product runs while the softmax still works on the current tile.  A
  // 128x64x16 product costs about 3/4 of a 128x128x16 one on the tensor pipe.  (Three query
  // tiles of 64 keys also fit at head_dim 64; measured, they ran no faster per query tile
  // and lost more to the last wave of CTAs.)
  static constexpr int NQ = 2;
  static constexpr int BN = HD == 64 ? 128 : 64;
  // warps: 4 per query tile (softmax), then the TMA producer, then three MMA issuers (the
  // first also owns the tensor memory)
  static constexpr int W_PROD = 4 * NQ;
  static constexpr int W_ISS = W_PROD + 1;
  static constexpr int kIssuers = 3;
  static constexpr int kThreads = 32 * (W_PROD + 4);
  static constexpr int kLaunchRegs = (kRegFile / kThreads) & ~7;  // the allocation granule is 8
  // setmaxnreg: the producer/issuer warpgroup gives registers back, the softmax warpgroups
  // take them (a softmax thread holds its row of S and P)
  static constexpr int kLowRegs = 72;
  static constexpr int kHighRegs = 216;
  static_assert(NQ * 128 * kHighRegs + 128 * kLowRegs <= kThreads * kLaunchRegs, "register split exceeds the launch");
  static constexpr int KCH = HD / 64;                    // 128-byte column chunks
  static constexpr int STAGES = 4;
  static constexpr int Q_CHUNK = BM * 128;               // one 64-column chunk of a Q tile
  static constexpr int KV_CHUNK = BN * 128;              // one 64-column chunk of a K or V tile
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  // When all of it fits, P has its own tensor-memory columns; otherwise P is written over
  // S_g.  The wider of the S and O regions comes first, so every region starts at a
  // multiple of its own width.
  static constexpr bool SEP_P = NQ * BN + NQ * (BN / 2) + NQ * HD <= kTmemCols;
  static constexpr bool O_FIRST = HD >= BN;
  static constexpr int COL_S = O_FIRST ? NQ * HD : 0;
  static constexpr int COL_P = SEP_P ? COL_S + NQ * BN : COL_S;
  static constexpr int P_STRIDE = SEP_P ? BN / 2 : BN;
  static constexpr int COL_O = O_FIRST ? 0 : (SEP_P ? COL_P + NQ * (BN / 2) : NQ * BN);
  static_assert(BN % 32 == 0 && (BN / 16 == 4 || BN / 16 == 8), "key tile width");
  // Issue split (see the MMA issuers), so that each issuing warp issues the same number of
  // products per key tile: one warp per query tile for whichever product has more
  // instructions (HD / 16 for S against BN / 16 for PV), one warp for the other product of
  // both tiles.
  enum Split { kSPerTile, kPVPerTile };
  static constexpr Split SPLIT = HD > BN ? kSPerTile : kPVPerTile;
  static_assert(NQ == 2, "the issue split assumes two query tiles (three issuing warps)");
  static constexpr int KV_EMPTY_ARRIVALS = SPLIT == kSPerTile ? 1 : NQ;  // PV-issuing warps
  static_assert((O_FIRST ? COL_P + NQ * P_STRIDE : COL_O + NQ * HD) <= kTmemCols, "tensor memory budget");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  // k_full[S], v_full[S], kv_empty[S], q_full[NQ], s_full[NQ], s_free[NQ], p_full[NQ], o_done[NQ], fin
  static constexpr int N_BAR = 3 * STAGES + 5 * NQ + 1;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
  // rows of each stage's key tile that are keys (several-slot instantiation: written by the
  // producer, read by the softmax warps)
  static constexpr int OFF_REM = OFF_MISC + 16;
  static constexpr int BYTES = OFF_REM + STAGES * 4;
  static constexpr int ALLOC = BYTES + 1024;             // room to align the base to 1 KB
  static_assert(ALLOC <= 227 * 1024, "shared memory budget");
};

struct Params {
  const __nv_bfloat16* q;  // raw window queries (bf16)
  const __nv_bfloat16* residual;
  __nv_bfloat16* out;
  int64_t n_win;
  int64_t cache_len;
  int32_t hidden;
  int32_t n_qpairs;
  int32_t n_ct;  // cache key tiles
  int32_t n_wt;  // window key tiles
  float scale_log2;
  uint32_t flags;
  uint32_t* status;
  BlockTable bt;
};

// Cache segments of the MULTI instantiation: segment s is rows [seg_row[s], seg_row[s] +
// seg_len[s]) of the cache tensors and key tiles [seg_tile0[s], seg_tile0[s + 1]).
struct SegParams {
  int32_t n_seg;
  int32_t seg_tile0[DP_MAX_SLOTS + 1];
  int32_t seg_row[DP_MAX_SLOTS];
  int32_t seg_len[DP_MAX_SLOTS];
};

// Cache tile j (< the cache tile count) -> its segment: the last s whose first tile is <= j.
__device__ __forceinline__ int seg_of_tile(const SegParams& sp, int j) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < DP_MAX_SLOTS; ++i) s += (i < sp.n_seg && j >= sp.seg_tile0[i]) ? 1 : 0;
  return s;
}

__device__ __forceinline__ float4 ld_f4(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <int HD, bool F16, bool MULTI>
__global__ void __launch_bounds__(Layout<HD>::kThreads, 1)
    window_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                          const __grid_constant__ CUtensorMap tm_kw, const __grid_constant__ CUtensorMap tm_vw,
                          const Params p, const __grid_constant__ SegParams sp) {
  using L = Layout<HD>;
  constexpr int BN = L::BN;
  constexpr int NQ = L::NQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qpair = blockIdx.x % p.n_qpairs;   // consecutive CTAs share a head (K/V reuse in L2)
  const int head = blockIdx.x / p.n_qpairs;
  const int n_tiles = p.n_ct + p.n_wt;

  const uint32_t bar0 = sb + L::OFF_BAR;
  auto k_full = [&](int s) { return bar0 + 8u * s; };
  auto v_full = [&](int s) { return bar0 + 8u * (L::STAGES + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (2 * L::STAGES + s); };
  auto q_full = [&](int g) { return bar0 + 8u * (3 * L::STAGES + g); };
  auto s_full = [&](int g) { return bar0 + 8u * (3 * L::STAGES + NQ + g); };
  auto s_free = [&](int g) { return bar0 + 8u * (3 * L::STAGES + 2 * NQ + g); };
  auto p_full = [&](int g) { return bar0 + 8u * (3 * L::STAGES + 3 * NQ + g); };
  auto o_done = [&](int g) { return bar0 + 8u * (3 * L::STAGES + 4 * NQ + g); };
  const uint32_t fin = bar0 + 8u * (3 * L::STAGES + 5 * NQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), L::KV_EMPTY_ARRIVALS);  // one arrival from each PV-issuing warp
    }
    for (int g = 0; g < NQ; ++g) {
      mbar_init(q_full(g), 128);
      mbar_init(s_full(g), 1);
      mbar_init(s_free(g), 128);
      mbar_init(p_full(g), 128);
      mbar_init(o_done(g), 1);
    }
    mbar_init(fin, L::kIssuers);  // one arrival from each MMA issuer
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == L::W_ISS) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == L::W_PROD && lane == 0) {
    tma_prefetch_desc(&tm_kc);
    tma_prefetch_desc(&tm_vc);
    tma_prefetch_desc(&tm_kw);
    tma_prefetch_desc(&tm_vw);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= L::W_PROD) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(L::kLowRegs));
  if (warp == L::W_PROD) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      const bool skip_loads = (p.flags & DP_TEST_SKIP_KV_LOADS) != 0;  // failure-path test hook
      for (int j = 0; j < n_tiles && !skip_loads; ++j) {
        const int st = j % L::STAGES;
        const int use = j / L::STAGES;
        if (use > 0 && !mbar_wait(kv_empty(st), (use - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_EMPTY)) break;
        const bool cache = j < p.n_ct;
        const CUtensorMap* mk = cache ? &tm_kc : &tm_kw;
        const CUtensorMap* mv = cache ? &tm_vc : &tm_vw;
        int row = (cache ? j : j - p.n_ct) * BN;
        if constexpr (MULTI) {
          int rem = static_cast<int>(p.n_win - static_cast<int64_t>(j - p.n_ct) * BN);
          if (cache) {
            const int sg = seg_of_tile(sp, j);
            row = pick(sp.seg_row, sg) + (j - pick(sp.seg_tile0, sg)) * BN;
            rem = pick(sp.seg_len, sg) - (j - pick(sp.seg_tile0, sg)) * BN;
          }
          // published before the arrive (release) that the softmax's test of k_full acquires
          reinterpret_cast<volatile int*>(smem + L::OFF_REM)[st] = rem < BN ? rem : BN;
        }
        mbar_arrive_expect_tx(k_full(st), L::KV_BYTES);
#pragma unroll
        for (int c = 0; c < L::KCH; ++c)
          tma_load_2d(sb + L::OFF_K + st * L::KV_BYTES + c * L::KV_CHUNK, mk, head * HD + c * 64, row, k_full(st));
        mbar_arrive_expect_tx(v_full(st), L::KV_BYTES);
#pragma unroll
        for (int c = 0; c < L::KCH; ++c)
          tma_load_2d(sb + L::OFF_V + st * L::KV_BYTES + c * L::KV_CHUNK, mv, head * HD + c * 64, row, v_full(st));
        issued = j + 1;
      }
      // every copy this CTA issued must land before its shared memory is released
      const int first = issued > L::STAGES ? issued - L::STAGES : 0;
      for (int j = first; j < issued; ++j) {
        mbar_drain_wait(k_full(j % L::STAGES), (j / L::STAGES) & 1, p.status);
        mbar_drain_wait(v_full(j % L::STAGES), (j / L::STAGES) & 1, p.status);
      }
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issuers
    // Products: S_g(t) = Q_g K_t^T needs K_t and S_g(t-1) consumed (read by the softmax when
    // P has its own columns; PV_g(t-1) complete when P is written over S_g); O_g += P_g(t) V_t
    // needs P_g(t) and V_t and releases the K/V stage.  A tcgen05.mma holds its issuing
    // thread while the tensor pipe's queue is full, so a warp's barrier tests and commits run
    // in series with the execution of its own products.  Three warps on three SM
    // sub-partitions therefore share the issuing, split so that each issues the same number
    // of products per key tile:
    //   head_dim 64 (4 S and 8 PV products per query tile): warp 9 S for both query
    //     tiles, warp 10 + g PV_g;
    //   head_dim 128 (8 S and 4 PV products per query tile): warp 9 + g S_g, warp 11 PV
    //     for both query tiles.
    // Each issuer waits with bounded waits and commits its own products.
    constexpr uint32_t idS = idesc_f32acc(Operand<F16>::kFmt, BM, BN, false);
    constexpr uint32_t idPV = idesc_f32acc(Operand<F16>::kFmt, BM, HD, true);
    auto wait = [&](uint32_t bar, uint32_t parity, uint32_t code) {
      return mbar_wait(bar, parity, abort, p.status, code);
    };
    // two waits with one overlapped fast path
    auto wait2 = [&](uint32_t b0, uint32_t p0, uint32_t c0, uint32_t b1, uint32_t p1, uint32_t c1) {
      return mbar_test_wait2(b0, p0, b1, p1) || (wait(b0, p0, c0) && wait(b1, p1, c1));
    };
    // Descriptors are built once; each MMA adds a compile-time offset to the 14-bit start
    // address field (16-byte units; every address stays below 2^18 bytes, so the sum never
    // carries out of the field).
    const uint64_t dq0 = sdesc_sw128(sb + L::OFF_Q, 16, 1024);
    const uint64_t dk0 = sdesc_sw128(sb + L::OFF_K, 16, 1024);
    const uint64_t dv0 = sdesc_sw128(sb + L::OFF_V, L::KV_CHUNK, 1024);
    bool ok = wait(q_full(0), 0, DEV_ERR_TIMEOUT_Q) && wait(q_full(1), 0, DEV_ERR_TIMEOUT_Q);
    // S_g(t) into S_g's columns (the caller has waited for K_t and for S_g(t-1) to be free)
    auto mma_s = [&](int st, int g) {
      tc_fence_after();
      const uint64_t dq = dq0 + static_cast<uint64_t>((g * L::Q_BYTES) >> 4);
      const uint64_t dk = dk0 + static_cast<uint64_t>((st * L::KV_BYTES) >> 4);
      const uint32_t d = tmem + L::COL_S + g * BN;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * L::Q_CHUNK + (kk & 3) * 32) >> 4);
        const uint64_t okv = static_cast<uint64_t>(((kk >> 2) * L::KV_CHUNK + (kk & 3) * 32) >> 4);
        mma_ss(d, dq + oq, dk + okv, idS, kk > 0);
      }
      mma_commit(s_full(g));
    };
    // O_g += P_g(t) V_t (the caller has waited for P_g(t) and V_t)
    auto mma_pv = [&](int t, int st, int g) {
      tc_fence_after();
      const uint64_t dv = dv0 + static_cast<uint64_t>((st * L::KV_BYTES) >> 4);
      const uint32_t pa = tmem + L::COL_P + g * L::P_STRIDE;
      const uint32_t d = tmem + L::COL_O + g * HD;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk)
        mma_ts(d, pa + kk * 8, dv + static_cast<uint64_t>((kk * 2048) >> 4), idPV, (t > 0 || kk > 0) ? 1u : 0u);
      mma_commit(o_done(g));
    };
    const int iw = warp - L::W_ISS;  // issuing warp 0..2
    if constexpr (L::SPLIT == L::kSPerTile) {
      if (iw < NQ) {
        const int g = iw;
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int st = t % L::STAGES;
          const uint32_t kpar = (t / L::STAGES) & 1;
          // both phases have normally completed: one overlapped test usually settles it
          if (t > 0)
            ok = wait2(L::SEP_P ? s_free(g) : o_done(g), (t - 1) & 1, L::SEP_P ? DEV_ERR_TIMEOUT_S : DEV_ERR_TIMEOUT_O,
                       k_full(st), kpar, DEV_ERR_TIMEOUT_KV);
          else
            ok = wait(k_full(st), kpar, DEV_ERR_TIMEOUT_KV);
          if (!ok) break;
          mma_s(st, g);
        }
      } else {
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int st = t % L::STAGES;
#pragma unroll 1
          for (int g = 0; g < NQ; ++g) {
            ok = wait(p_full(g), t & 1, DEV_ERR_TIMEOUT_P) &&
                 (g > 0 || wait(v_full(st), (t / L::STAGES) & 1, DEV_ERR_TIMEOUT_KV));
            if (!ok) break;
            mma_pv(t, st, g);
          }
          if (ok) mma_commit(kv_empty(st));  // after the stage's last PV product
        }
      }
    } else {
      if (iw == 0) {
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int st = t % L::STAGES;
#pragma unroll 1
          for (int g = 0; g < NQ; ++g) {
            if (t > 0) {
              ok = L::SEP_P ? wait(s_free(g), (t - 1) & 1, DEV_ERR_TIMEOUT_S)
                            : wait(o_done(g), (t - 1) & 1, DEV_ERR_TIMEOUT_O);
              if (!ok) break;
            }
            if (g == 0) {
              ok = wait(k_full(st), (t / L::STAGES) & 1, DEV_ERR_TIMEOUT_KV);
              if (!ok) break;
            }
            mma_s(st, g);
          }
        }
      } else {
        const int g = iw - 1;
        for (int t = 0; ok && t < n_tiles; ++t) {
          const int st = t % L::STAGES;
          ok = wait(p_full(g), t & 1, DEV_ERR_TIMEOUT_P) && wait(v_full(st), (t / L::STAGES) & 1, DEV_ERR_TIMEOUT_KV);
          if (!ok) break;
          mma_pv(t, st, g);
          mma_commit(kv_empty(st));
        }
      }
    }
    if (warp >= L::W_ISS) {
      // every product this warp issued completes before TMEM is released
      mma_commit(fin);
      mbar_drain_wait(fin, 0, p.status);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(L::kHighRegs));
    // ------------------------------------------------------------ softmax warpgroups
    const int g = warp >> 2;                       // query tile of this warpgroup
    const int t = threadIdx.x & 127;               // row within the tile
    const int64_t qrow = static_cast<int64_t>(qpair) * (NQ * BM) + g * BM + t;
    const bool row_ok = qrow < p.n_win;
    const int blk = row_ok ? block_of_row(p.bt, qrow) : 0;
    const float* modb = block_mod(p.bt, blk);

    // prologue: modulated query row -> swizzled K-major shared-memory tile
    {
      uint8_t* sq = smem + L::OFF_Q + g * L::Q_BYTES;
      const uint4* src = reinterpret_cast<const uint4*>(p.q + qrow * p.hidden + head * HD);
      const float* shift = modb + head * HD;
      const float* scale = modb + p.hidden + head * HD;
#pragma unroll 4
      for (int c = 0; c < HD / 8; ++c) {
        uint4 outv = make_uint4(0, 0, 0, 0);
        if (row_ok) {
          const uint4 raw = src[c];
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
          float xf[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(x2[e]);
            xf[2 * e] = f.x;
            xf[2 * e + 1] = f.y;
          }
          if (p.flags & DP_MOD_Q) {
            const float4 sh0 = ld_f4(shift + c * 8), sh1 = ld_f4(shift + c * 8 + 4);
            const float4 sc0 = ld_f4(scale + c * 8), sc1 = ld_f4(scale + c * 8 + 4);
            const float sh[8] = {sh0.x, sh0.y, sh0.z, sh0.w, sh1.x, sh1.y, sh1.z, sh1.w};
            const float sc[8] = {sc0.x, sc0.y, sc0.z, sc0.w, sc1.x, sc1.y, sc1.z, sc1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) xf[e] = fmaf(xf[e], 1.0f + sc[e], sh[e]);
          }
          outv = make_uint4(Operand<F16>::pack(xf[0], xf[1]), Operand<F16>::pack(xf[2], xf[3]),
                            Operand<F16>::pack(xf[4], xf[5]), Operand<F16>::pack(xf[6], xf[7]));
        }
        const int chunk = c >> 3, w = c & 7;
        *reinterpret_cast<uint4*>(sq + chunk * L::Q_CHUNK + t * 128 + ((w ^ (t & 7)) << 4)) = outv;
      }
      fence_proxy_async_smem();
      mbar_arrive(q_full(g));
    }

    const uint32_t trow = tmem + ((static_cast<uint32_t>(warp & 3) * 32u) << 16);
    const uint32_t s_col = L::COL_S + g * BN;
    constexpr int NCH = BN / 32;  // 32-column chunks of an S row
    constexpr int NG = BN / 16;   // max chains
    const uint32_t p_col = L::COL_P + g * L::P_STRIDE;
    const uint32_t o_col = L::COL_O + g * HD;
    const uint64_t sl2 = f32x2(p.scale_log2, p.scale_log2);
    float m_ref = -INFINITY;
    float l_sum = 0.0f;
    bool ok = true;

    for (int j = 0; j < n_tiles; ++j) {
      ok = mbar_wait(s_full(g), j & 1, abort, p.status, DEV_ERR_TIMEOUT_S);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[NCH][32];
#pragma unroll
      for (int i = 0; i < NCH; ++i) tmem_ld32(trow + s_col + i * 32, sr[i]);
      tmem_wait_ld();
      if constexpr (L::SEP_P) {
        // S is in registers: the tensor core may overwrite it with the next tile's S
        tc_fence_before();
        mbar_arrive(s_free(g));
      }
      const int64_t key0 = (j < p.n_ct) ? static_cast<int64_t>(j) * BN : static_cast<int64_t>(j - p.n_ct) * BN;
      int64_t rem = ((j < p.n_ct) ? p.cache_len : p.n_win) - key0;
      if constexpr (MULTI) {
        // rows of this tile that are keys, as the producer published them for the stage; the
        // stage's k_full phase for tile j completed before S(j) could (and it is not refilled
        // before this tile's P is stored), so the test succeeds and orders the read after the
        // producer's write
        const int st = j % L::STAGES;
        if (mbar_test_wait(k_full(st), (j / L::STAGES) & 1))
          rem = reinterpret_cast<volatile int*>(smem + L::OFF_REM)[st];
      }
      if (rem < BN) {  // last tile of a segment: keys beyond it get -inf (TMA filled them with 0)
        const int valid = static_cast<int>(rem);
#pragma unroll
        for (int i = 0; i < NCH; ++i)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (i * 32 + c >= valid) sr[i][c] = 0xff800000u;
      }
      // row max: NG independent chains of 3-input max (short dependency chains)
      float mc[NG];
#pragma unroll
      for (int h = 0; h < NG; ++h) {
        const uint32_t* r = &sr[h >> 1][(h & 1) * 16];
        float m = fmaxf(__uint_as_float(r[0]), __uint_as_float(r[15]));
#pragma unroll
        for (int c = 1; c < 15; c += 2) m = fmax3(m, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
        mc[h] = m;
      }
      float mx;
      if constexpr (NG == 8)
        mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
      else
        mx = fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
      const float m_new = fmaxf(m_ref, mx * p.scale_log2);
      if (j == 0) {
        m_ref = m_new;
      } else {
        const bool need = m_new > m_ref + kRescaleLog2;
        const bool any_need = __any_sync(0xffffffffu, need);
        if (any_need) {
          // PV(j-1) must be complete before O is rescaled
          ok = mbar_wait(o_done(g), (j - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_O);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float f = need ? ex2_approx(m_ref - m_new) : 1.0f;
#pragma unroll
          for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t orr[32];
            tmem_ld32(trow + o_col + c0, orr);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * f);
            tmem_st32(trow + o_col + c0, orr);
          }
          tmem_wait_st();
          if (need) {
            l_sum *= f;
            m_ref = m_new;
          }
        }
      }
      // P = exp2(s * scale * log2(e) - m_ref): packed FMA, exp2 on the MUFU unit or (for
      // the PolyPairs columns) on the FMA pipe, packed adds for the row sum
      const uint64_t nm2 = f32x2(-m_ref, -m_ref);
      const uint64_t magic2 = f32x2(kRoundMagic, kRoundMagic);
      const uint64_t nmagic2 = f32x2(-kRoundMagic, -kRoundMagic);
      const uint64_t neg1_2 = f32x2(-1.0f, -1.0f);
      const uint64_t c0_2 = f32x2(kPolyC0, kPolyC0), c1_2 = f32x2(kPolyC1, kPolyC1);
      const uint64_t c2_2 = f32x2(kPolyC2, kPolyC2), c3_2 = f32x2(kPolyC3, kPolyC3);
      uint64_t acc0 = f32x2(0.0f, 0.0f), acc1 = acc0;
      uint32_t pk[NCH][16];  // P stays in registers until PV(j-1) has released its columns
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint64_t x = ffma2(f32x2(__uint_as_float(sr[i][2 * c]), __uint_as_float(sr[i][2 * c + 1])), sl2, nm2);
          float x0, x1;
          f32x2_split(x, x0, x1);
          float a, b;
          if ((PolyPairs<HD>::kMask >> c) & 1u) {
            const uint64_t xc = f32x2(fmaxf(x0, kPolyMinX), fmaxf(x1, kPolyMinX));
            const uint64_t t = fadd2(xc, magic2);        // low mantissa bits hold round(x)
            const uint64_t f = ffma2(fadd2(t, nmagic2), neg1_2, xc);  // x - round(x)
            uint64_t q = ffma2(c3_2, f, c2_2);
            q = ffma2(q, f, c1_2);
            q = ffma2(q, f, c0_2);
            float q0, q1, t0, t1;
            f32x2_split(q, q0, q1);
            f32x2_split(t, t0, t1);
            a = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
            b = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
          } else {
            a = ex2_approx(x0);
            b = ex2_approx(x1);
          }
          const uint64_t ab = f32x2(a, b);
          if (c & 1)
            acc1 = fadd2(acc1, ab);
          else
            acc0 = fadd2(acc0, ab);
          pk[i][c] = Operand<F16>::pack_p(a, b);
        }
      }
      if constexpr (L::SEP_P) {
        if (j > 0) {
          // P(j-1) in these columns must have been read by PV(j-1); by now it has been
          ok = mbar_wait(o_done(g), (j - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_O);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
      }
#pragma unroll
      for (int i = 0; i < NCH; ++i) tmem_st16(trow + p_col + i * 16, pk[i]);
      {
        const uint64_t acc = fadd2(acc0, acc1);
        float a0, a1;
        f32x2_split(acc, a0, a1);
        l_sum += a0 + a1;
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(g));
    }

    // epilogue: O / l, gate, residual, bf16 store
    if (ok && n_tiles > 0) {
      ok = mbar_wait(o_done(g), (n_tiles - 1) & 1, abort, p.status, DEV_ERR_TIMEOUT_O);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_sum;
      const float* gate = modb + 2 * p.hidden + head * HD;
      const bool do_gate = (p.flags & DP_GATE_OUT) != 0;
#pragma unroll
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t orr[32];
        tmem_ld32(trow + o_col + c0, orr);
        tmem_wait_ld();
        if (row_ok) {
          float vals[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) vals[c] = __uint_as_float(orr[c]) * inv_l;
          if (do_gate) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 gv = ld_f4(gate + c0 + c);
              vals[c] *= gv.x;
              vals[c + 1] *= gv.y;
              vals[c + 2] *= gv.z;
              vals[c + 3] *= gv.w;
            }
          }
          if (p.residual) {
            const uint4* rs = reinterpret_cast<const uint4*>(p.residual + qrow * p.hidden + head * HD + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 r = rs[c];
              const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 rf = __bfloat1622float2(r2[e]);
                vals[c * 8 + 2 * e] += rf.x;
                vals[c * 8 + 2 * e + 1] += rf.y;
              }
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(p.out + qrow * p.hidden + head * HD + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            dst[c] = make_uint4(pack_bf16x2(vals[c * 8 + 0], vals[c * 8 + 1]), pack_bf16x2(vals[c * 8 + 2], vals[c * 8 + 3]),
                                pack_bf16x2(vals[c * 8 + 4], vals[c * 8 + 5]), pack_bf16x2(vals[c * 8 + 6], vals[c * 8 + 7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::W_ISS) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

template <int HD, bool F16, bool MULTI>
cudaError_t launch_hd(const AttnArgs& a, cudaStream_t s) {
  using L = Layout<HD>;
  CUtensorMap tkc, tvc, tkw, tvw;
  constexpr int BN = L::BN;
  if (!encode_tmap_16(&tkw, a.k, a.n_win, a.hidden, BN, F16) || !encode_tmap_16(&tvw, a.v, a.n_win, a.hidden, BN, F16))
    return cudaErrorInvalidValue;
  // one range: the segment's own rows (its first row is the map's row 0); several: the ring
  const CacheSegs& g = a.segs;
  const int64_t row_bytes = static_cast<int64_t>(a.hidden) * 2;
  const char* ck = static_cast<const char*>(a.cache_k) + (MULTI ? 0 : static_cast<int64_t>(g.row[0]) * row_bytes);
  const char* cv = static_cast<const char*>(a.cache_v) + (MULTI ? 0 : static_cast<int64_t>(g.row[0]) * row_bytes);
  const int64_t map_rows = MULTI ? a.cache_rows : a.cache_len;
  if (a.cache_len > 0) {
    if (!encode_tmap_16(&tkc, ck, map_rows, a.hidden, BN, F16) || !encode_tmap_16(&tvc, cv, map_rows, a.hidden, BN, F16))
      return cudaErrorInvalidValue;
  } else {
    tkc = tkw;
    tvc = tvw;
  }
  SegParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.n_seg = g.n;
  for (int i = 0; i < DP_MAX_SLOTS; ++i) {
    const bool in = i < g.n;
    sp.seg_row[i] = in ? g.row[i] : 0;
    sp.seg_len[i] = in ? g.len[i] : 0;
    sp.seg_tile0[i + 1] = sp.seg_tile0[i] + (in ? (g.len[i] + BN - 1) / BN : 0);
  }
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.residual = static_cast<const __nv_bfloat16*>(a.residual);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.n_win = a.n_win;
  p.cache_len = a.cache_len;
  p.hidden = a.hidden;
  p.n_qpairs = static_cast<int32_t>((a.n_win + L::NQ * BM - 1) / (L::NQ * BM));
  p.n_ct = MULTI ? sp.seg_tile0[DP_MAX_SLOTS] : static_cast<int32_t>((a.cache_len + BN - 1) / BN);
  p.n_wt = static_cast<int32_t>((a.n_win + BN - 1) / BN);
  p.scale_log2 = a.softmax_scale * 1.4426950408889634f;
  p.flags = a.flags;
  p.status = a.status;
  p.bt = a.bt;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<bool> attr_set[64];  // per instantiation and device (concurrent first calls both set it)
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(window_attn_tc_kernel<HD, F16, MULTI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::ALLOC);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc waits for registers the launch did not provide: refuse to launch if
    // the compiled register count is below the split's assumption.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, window_attn_tc_kernel<HD, F16, MULTI>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < L::kLaunchRegs) return cudaErrorInvalidConfiguration;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t grid = static_cast<int64_t>(p.n_qpairs) * a.n_heads;
  window_attn_tc_kernel<HD, F16, MULTI><<<static_cast<unsigned>(grid), L::kThreads, L::ALLOC, s>>>(tkc, tvc, tkw, tvw,
                                                                                                  p, sp);
  return cudaGetLastError();
}

}  // namespace

bool encode_tmap_16(void* tmap, const void* base, int64_t rows, int hidden, int box_rows, bool f16) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(hidden) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(static_cast<CUtensorMap*>(tmap), f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_attention_tc(const AttnArgs& a, bool f16_features, cudaStream_t s) {
  const bool multi = a.segs.n > 1;
  if (a.head_dim == 64) {
    if (multi) return f16_features ? launch_hd<64, true, true>(a, s) : launch_hd<64, false, true>(a, s);
    return f16_features ? launch_hd<64, true, false>(a, s) : launch_hd<64, false, false>(a, s);
  }
  if (a.head_dim == 128) {
    if (multi) return f16_features ? launch_hd<128, true, true>(a, s) : launch_hd<128, false, true>(a, s);
    return f16_features ? launch_hd<128, true, false>(a, s) : launch_hd<128, false, false>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dp
