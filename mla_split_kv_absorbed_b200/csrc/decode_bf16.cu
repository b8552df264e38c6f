// Steps A2-A8 for a bf16 latent cache (kernel to follow; FP8 path first).
#include "kernels.cuh"

namespace mla {

cudaError_t launch_decode_bf16(const DecodeArgs&, const CUtensorMap&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace mla
