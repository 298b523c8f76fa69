// Launchers of the tcgen05 / TMEM / TMA kernels for sm_100a (bf16 path).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace rest {

// 2-D bf16 TMA descriptor over a row-major [rows, cols] array with a row stride
// of `stride` elements; box of box_cols x box_rows; swizzle 128 or 64 bytes.
bool make_tmap_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, long long stride,
                    int box_cols, int box_rows, int swizzle_bytes);

// True when the tensor-core GEMM handles this shape and epilogue.
bool sm100_gemm_supported(const GemmArgs& a);
cudaError_t launch_gemm_sm100(const GemmArgs& a, cudaStream_t s, int32_t* err);

// True when the tensor-core attention kernels handle this head_dim.
bool sm100_attn_supported(int head_dim);
// Query rows per work item of the tensor-core attention kernels.
int sm100_attn_tile_rows(int head_dim);
cudaError_t launch_enc_attn_sm100(int head_dim, const EncAttnArgs& a, cudaStream_t s, int32_t* err);
cudaError_t launch_dec_attn_sm100(int head_dim, const DecAttnArgs& a, cudaStream_t s, int32_t* err);
// Backward of the causal attention core (head_dim 32 or 64): dq (zeroed by the
// caller, accumulated with atomics), dk and dv.
cudaError_t launch_attn_bwd_sm100(int head_dim, const AttnBwdArgs& a, cudaStream_t s, int32_t* err);

// Failure-detection self-test: n_ctas CTAs wait on a barrier nothing completes;
// CTA 0 gives up after limit_cycles and sets REST_ERR_TIMEOUT, the others on seeing it.
cudaError_t launch_wait_timeout(int n_ctas, long long limit_cycles, int32_t* err, cudaStream_t s);

}  // namespace rest
