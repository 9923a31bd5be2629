// Internal interfaces between the C ABI (dp_api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

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

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* cache_k;
  const void* cache_v;
  const void* residual;
  void* out;
  int64_t n_win;
  int64_t cache_len;
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

// Host-side helper: encode a 2-D 16-bit (f16 or bf16) tensor map [rows][hidden] with a
// {64 columns, box_rows rows} box and 128-byte swizzle (defined in dp_attn_tc.cu).
bool encode_tmap_16(void* tmap, const void* base, int64_t rows, int hidden, int box_rows, bool f16);

}  // namespace dp
