// Launchers of the tcgen05 / TMEM / TMA kernels for sm_100a (bf16 path).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace rest {

// True when the tensor-core GEMM handles this shape and epilogue.
bool sm100_gemm_supported(const GemmArgs& a);
cudaError_t launch_gemm_sm100(const GemmArgs& a, cudaStream_t s, int32_t* err);

// True when the tensor-core attention kernels handle this head_dim.
bool sm100_attn_supported(int head_dim);
cudaError_t launch_enc_attn_sm100(int head_dim, const EncAttnArgs& a, cudaStream_t s, int32_t* err);
cudaError_t launch_dec_attn_sm100(int head_dim, const DecAttnArgs& a, cudaStream_t s, int32_t* err);

}  // namespace rest
