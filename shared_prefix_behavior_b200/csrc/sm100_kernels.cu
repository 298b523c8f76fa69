// tcgen05 / TMEM / TMA kernels for sm_100a (bf16 path).
#include "sm100.h"

namespace rest {

bool sm100_attn_supported(int) { return false; }
cudaError_t launch_enc_attn_sm100(int, const EncAttnArgs&, cudaStream_t, int32_t*) { return cudaErrorNotSupported; }
cudaError_t launch_dec_attn_sm100(int, const DecAttnArgs&, cudaStream_t, int32_t*) { return cudaErrorNotSupported; }

}  // namespace rest
