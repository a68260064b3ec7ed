// k_attn_tc.cu — attention on the sm_100a tensor cores (placeholder: routes
// to the CUDA-core kernel until the tcgen05 version is in place).
#include "wd_internal.cuh"

namespace wd {
wd_status attention_tc(const AttnArgs<bf16>& a, cudaStream_t st) { return attention_simt<bf16>(a, st); }
}  // namespace wd
