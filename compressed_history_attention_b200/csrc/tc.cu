// Tensor-core kernels (tcgen05 + TMEM).  Shapes without one fall back to the
// fp32 CUDA-core kernels.
#include "tc.cuh"

namespace nanokv {

bool tc_encode_supported(const Codec &) { return false; }
bool tc_low_supported(const Codec &, const Codec &) { return false; }

cudaError_t tc_encode(const Codec &, const void *, int64_t, uint8_t *, uint8_t *, void *,
                      cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_attend_low(const void *, int64_t, const Codec &, const Codec &, const Hist &,
                          const Hist &, int64_t, int64_t, float, Part, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace nanokv
