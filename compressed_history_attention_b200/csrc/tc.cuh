// Tensor-core (tcgen05 / TMEM) kernels for sm_100a: launchers and the shape
// predicates that decide whether a tensor-core kernel exists for a call.
#pragma once
#include "common.cuh"

namespace nanokv {

bool tc_encode_supported(const Codec &c);
bool tc_full_supported(const Codec &ck, const Codec &cv);
bool tc_low_supported(const Codec &ck, const Codec &cv);
bool tc_dense_supported(int prec, int d);

cudaError_t tc_encode(const Codec &c, const void *x, int64_t T, uint8_t *ids, uint8_t *codes,
                      void *scales, cudaStream_t st);
cudaError_t tc_attend_full(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                           const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                           Part out, cudaStream_t st);
cudaError_t tc_attend_low(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                          const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                          Part out, cudaStream_t st);
cudaError_t tc_attend_dense(const void *q, int64_t Tq, int H, int d, const void *k, const void *v,
                            int64_t T, float tau, Part out, cudaStream_t st);

unsigned *error_word_ptr();

}  // namespace nanokv
