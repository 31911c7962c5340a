// Tensor-core (tcgen05 / TMEM) kernels for sm_100a: launchers and the shape
// predicates that decide whether a tensor-core kernel exists for a call.
#pragma once
#include "common.cuh"

namespace nanokv {

bool tc_encode_supported(const Codec &c);
bool tc_full_supported(const Codec &ck, const Codec &cv);
bool tc_low_supported(const Codec &ck, const Codec &cv);
// larger codecs (r in {128, 256, 384}, up to 256 centers): a 2-CTA kernel
bool tc_low_pair_supported(const Codec &ck, const Codec &cv);
bool tc_dense_supported(int prec, int d);

// encodes nbranch (1 or 2) branches with equal C and r in one launch
cudaError_t tc_encode_pair(const Codec *c, const void *const *x, int64_t T, uint8_t *const *ids,
                           uint8_t *const *codes, void *const *scales, int nbranch, cudaStream_t st);
size_t codec_aux_bytes(const Codec &c);
cudaError_t codec_prepare(const Codec &c, void *aux, cudaStream_t st);
// The full-dim kernel may split the history [t0, t0 + T) into nsplit
// contiguous ranges of whole key tiles (grid z), each writing its own fp32
// partial: split z at out.O + z * ostride, out.LSE + z * lstride.
constexpr int kMaxFullSplits = 6;
int tc_full_splits(int64_t Tq, int H, int d, int64_t T);
cudaError_t tc_attend_full(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                           const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                           Part out, int nsplit, size_t ostride, size_t lstride, cudaStream_t st,
                           bool pdl, HeadSel hs = HeadSel{nullptr, 0});
// Heads at a reduced attention dimension d_h (32, 64 or 96): the full-dim
// kernel at width d_h on the reduced queries [Tq, H*128] and the mapped
// decoder / centers (ck_red, cv_red), restoring its rows with the value maps
// W [H, 128, 128].  One history split.
bool tc_reduced_dim_ok(int d_h);
cudaError_t tc_attend_reduced(int d_h, const void *q_red, int64_t Tq, const Codec &ck_red, const Codec &cv_red,
                              const void *W, const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                              Part out, cudaStream_t st, HeadSel hs);
cudaError_t tc_attend_low(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                          const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                          Part out, cudaStream_t st, HeadSel hs = HeadSel{nullptr, 0});
cudaError_t tc_attend_low_pair(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                               const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                               Part out, cudaStream_t st, HeadSel hs = HeadSel{nullptr, 0});
cudaError_t tc_attend_dense(const void *q, int64_t Tq, int H, int d, const void *k, const void *v,
                            int64_t T, float tau, Part out, cudaStream_t st, bool pdl);

unsigned *error_word_ptr();

}  // namespace nanokv
