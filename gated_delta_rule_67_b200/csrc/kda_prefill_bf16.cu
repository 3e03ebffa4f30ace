// kda_prefill_bf16.cu -- bf16 chunked KDA prefill (tcgen05 path): placeholder
// until the tensor-core kernels land; reports "not supported".
#include "kda_common.cuh"

namespace kda {

size_t prefill_bf16_workspace_bytes(int, int, int, int, int, int) { return 0; }

cudaError_t launch_prefill_bf16(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                const __nv_bfloat16*, const __nv_bfloat16*, float, const float*,
                                __nv_bfloat16*, float*, int, int, int, int, int, int, void*, size_t,
                                cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kda
