// Internal interfaces between the C ABI (dp_api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <vector_types.h>

#include "dp.h"

namespace dp {

// Kernel-argument copy of dp_blocks (rows are int32 offsets into the window).
struct BlockTable {
  int32_t n_blocks;
  int32_t row_offset[DP_MAX_BLOCKS + 1];
  const float* mod[DP_MAX_BLOCKS];
};

// Block b owns rows [row_offset[b], row_offset[b+1]): the last b whose start is <= row.
// Unrolled over the table's fixed size so the kernel argument is never indexed at run time.
__host__ __device__ __forceinline__ int block_of_row(const BlockTable& t, int64_t row) {
  int b = 0;
#pragma unroll
  for (int i = 1; i < DP_MAX_BLOCKS; ++i) b += (i < t.n_blocks && row >= t.row_offset[i]) ? 1 : 0;
  return b;
}

// mod[b] selected with compile-time indices (see block_of_row).
__host__ __device__ __forceinline__ const float* block_mod(const BlockTable& t, int b) {
  const float* m = t.mod[0];
#pragma unroll
  for (int i = 1; i < DP_MAX_BLOCKS; ++i) m = (i == b) ? t.mod[i] : m;
  return m;
}

// The cache rows attention reads: segment s is rows [row[s], row[s] + len[s]) of cache_k /
// cache_v (one segment per cache slot read; zero segments when the cache is empty).
struct CacheSegs {
  int32_t n;
  int32_t row[DP_MAX_SLOTS];
  int32_t len[DP_MAX_SLOTS];
};

// Element i of a small kernel-argument array, selected with compile-time indices (a run-time
// index into a kernel argument would copy it to local memory).
template <int N>
__host__ __device__ __forceinline__ int32_t pick(const int32_t (&a)[N], int i) {
  int32_t v = a[0];
#pragma unroll
  for (int k = 1; k < N; ++k) v = (k == i) ? a[k] : v;
  return v;
}

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* cache_k;
  const void* cache_v;
  const void* residual;
  void* out;
  int64_t n_win;
  int64_t cache_len;    // total cache rows read (the sum of the segments' lengths)
  int64_t cache_rows;   // rows cache_k / cache_v hold (the extent the segments index into)
  CacheSegs segs;
  int32_t n_heads;
  int32_t head_dim;
  int32_t hidden;
  float softmax_scale;
  uint32_t flags;
  BlockTable bt;
  uint32_t* status;  // device status word
};

struct CopySeg {
  const void* src;
  void* dst;
  int64_t bytes;  // multiple of 16, both pointers 16-byte aligned
};
constexpr int kMaxCopySegs = 4;

// Tensor-core path: q, residual, out bf16; k, v, cache f16 (f16_features) or bf16.
cudaError_t launch_attention_tc(const AttnArgs& a, bool f16_features, cudaStream_t s);
cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t s);

// Records `msg` as this thread's dp_last_error_detail() and returns `s` (dp_api.cu).
dp_status set_error(dp_status s, const char* msg);
// x_dt -> y_dt: bf16 -> bf16, bf16 -> f16 (saturating), f16 -> f16, f32 -> f32.
cudaError_t launch_modulate(const void* const* src, void* const* dst, int nseg, int64_t n_rows,
                            int hidden, const BlockTable& bt, dp_dtype x_dt, dp_dtype y_dt, cudaStream_t s);
cudaError_t launch_copy(const CopySeg* segs, int nseg, cudaStream_t s);

// Frames idx[0 .. n_frames) of a pool ([frames][vec_per_frame] 16-byte vectors) copied in that
// order to dst0 and to dst1 (a queue slot and its mirror).
constexpr int kMaxGatherFrames = 16;
struct FrameGather {
  const uint4* pool;
  uint4* dst0;
  uint4* dst1;
  uint32_t vec_per_frame;
  int32_t n_frames;
  int32_t idx[kMaxGatherFrames];
};
cudaError_t launch_gather_frames(const FrameGather& g, cudaStream_t s);

// Linear layer on the tensor cores (dp_gemm.cu): y = a W^T + bias with a [m][k] bf16 and
// W [n][k] bf16, fp32 accumulation, then one of three epilogues.
enum GemmEpi {
  kEpiStore = 0,         // y0 [m][ld_y], bf16 or f16 (y_f16)
  kEpiQKV = 1,           // columns [0, s) -> y0 (q, bf16), [s, 2s) -> y1 (k, f16), [2s, 3s) -> y2 (v, f16)
  kEpiGateResidual = 2,  // y0 = residual + gate_b * (a W^T + bias), bf16; b = block of the row
  kEpiKV = 3,            // columns [0, s) -> y1 (k, f16), [s, 2s) -> y2 (v, f16)
};

struct GemmArgs {
  const void* a;
  const void* w;
  const float* bias;   // [n] or NULL
  int64_t m;
  int32_t n;           // multiple of 128
  int32_t k;           // multiple of 8
  int32_t epi;
  void* y0;
  void* y1;
  void* y2;
  int32_t ld_y;
  int32_t seg_cols;
  int32_t y_f16;
  const void* residual;
  BlockTable bt;
  uint32_t* status;
};

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s);

// Pre-norm and modulation (dp_modulate.cu): h = LN(x) * (1 + scale_b) + shift_b per row,
// LN without affine over the row's hidden channels in fp32; x and h bf16.
cudaError_t launch_ln_modulate(const void* x, void* h, int64_t n_rows, int hidden, float eps, const BlockTable& bt,
                               cudaStream_t s);

// Host-side helper: encode a 2-D 16-bit (f16 or bf16) tensor map [rows][hidden] with a
// {64 columns, box_rows rows} box and 128-byte swizzle (defined in dp_attn_tc.cu).
bool encode_tmap_16(void* tmap, const void* base, int64_t rows, int hidden, int box_rows, bool f16);

}  // namespace dp
