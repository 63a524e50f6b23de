// placeholder, replaced by the tcgen05 prefill kernel
#include "common.cuh"
namespace pkv {
cudaError_t launch_prefill_bf16(const PrefillParams&, cudaStream_t) { return cudaErrorNotSupported; }
}
