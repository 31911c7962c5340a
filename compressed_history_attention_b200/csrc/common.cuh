// Shared device helpers and the internal launcher interface of libnanokv.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

namespace nanokv {

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// INT4 nibble (two's complement) -> int
__device__ __forceinline__ int nib_lo(uint8_t b) { return (int)((int8_t)(b << 4) >> 4); }
__device__ __forceinline__ int nib_hi(uint8_t b) { return (int)((int8_t)b >> 4); }

// error-word bits (device error word, read by nanokv_check)
enum : unsigned { ERRW_TIMEOUT = 1u, ERRW_BOUNDS = 2u };

// ---------------------------------------------------------------------------
// internal argument bundles (plain pointers; no torch types anywhere)
// ---------------------------------------------------------------------------
struct Codec {
  int H, d, r, C;
  int prec;  // 0 = fp32 everywhere, 1 = bf16 params/io + fp16 scales
  const void *centers, *D, *E;
  const void *aux;  // optional derived encode tables (E c_j, |c_j|^2)
};
struct Hist {
  const uint8_t *ids, *codes;
  const void *scales;
};

enum Prec { PREC_F32 = 0, PREC_BF16 = 1 };

// The heads one history-kernel launch covers: all H (map == nullptr), or the
// n heads listed in the device array map (grid y indexes the list).
struct HeadSel {
  const int32_t *map;
  int n;
};

// fp32 partial output of one attention branch: O [Tq, H, d], LSE [H, Tq]
struct Part {
  float *O, *LSE;
};

constexpr int kMaxParts = 8;
struct PartList {
  const float *O[kMaxParts];
  const float *LSE[kMaxParts];
  int n;
};

// Gather of routed history tokens into contiguous compressed histories.
// A set is a list of segments: output tokens [dst, dst + cnt) are source
// tokens [src, src + cnt).  Up to 64 routed ranges give up to 65 segments of
// the complement.
constexpr int kMaxSegs = 65;
struct GatherSegs {
  int64_t src[kMaxSegs], dst[kMaxSegs], cnt[kMaxSegs];
  int n;
};
// How a routed call reads a head's low-dim tokens: full-dim (heads kept at
// full dimension), in the coefficient space (the low-dim kernels), or at a
// reduced attention dimension of 32, 64 or 96.
enum HeadClass : uint8_t { HC_FULL = 0, HC_LOW = 1, HC_R32 = 2, HC_R64 = 3, HC_R96 = 4, HC_COUNT = 5 };
struct GatherArgs {
  const uint8_t *ids[2], *codes[2], *scales[2];            // source history, [K / V]
  uint8_t *d_ids[2][2], *d_codes[2][2], *d_scales[2][2];   // destinations, [set][K / V]
  int64_t n_out[2];                                       // tokens per set (full-dim, low-dim)
  int row_bytes[2];                                       // packed code bytes per token, [K / V]
  int scale_bytes;                                        // 2 (fp16) or 4 (fp32)
  uint8_t head_class[256];                                // HeadClass of each head
  int H;
  int32_t *head_lists;  // [HC_COUNT + 1][H]: the heads of each class, in order; then all reduced heads
};
cudaError_t gather_launch(const GatherSegs &full, const GatherSegs &low, const GatherArgs &a, cudaStream_t st);

// Reduced attention dimension (lowdim.cu): mapped decoder rows [H*128, r]
// and centers [C, H*128] (bf16) of each branch, in a caller buffer.
struct LowdimTables {
  void *D[2], *cen[2];
};
struct HeadDims {
  uint8_t d[256];  // reduced attention dimension of each head (0: not reduced)
};
size_t lowdim_aux_bytes(const Codec &ck, const Codec &cv);
LowdimTables lowdim_tables(const Codec &ck, const Codec &cv, void *aux);
cudaError_t lowdim_prepare(const Codec &ck, const Codec &cv, const void *U, const void *W, void *aux,
                           cudaStream_t st);
cudaError_t reduce_queries(const void *q, int64_t Tq, int H, const void *U, HeadSel heads, const HeadDims &dims,
                           void *qred, cudaStream_t st);
// analytical maps [H, 128, 128] bf16 from a codec's decoder (bf16, d = 128)
cudaError_t lowdim_analytic(const Codec &c, void *maps, cudaStream_t st);

// Codec calibration (calibrate.cu): k-means centers, then the leading
// eigenvectors of the residual second moment.  Outputs in the tokens' dtype.
constexpr int kCalibSweeps = 30;  // Jacobi sweeps at most (stops once converged)
struct CalibArgs {
  const void *x;        // [N, J] tokens (fp32 or bf16, prec)
  int64_t N;
  int J, C, r, rounds, prec;
  const float *init;    // [C, J] initial centers
  void *centers, *D, *E;  // outputs [C, J], [J, r], [r, J]
  uint8_t *ids;         // [N] final assignment (workspace when the caller passes none)
  float *evals;         // [r] or nullptr
  float *cen32;          // workspace: fp32 centers
  double *S, *V;         // workspace: the second moment / its eigenvectors (fp64)
  void *rot;
  int *done;
};
size_t calibrate_workspace(int64_t N, int J, int C);
void calibrate_carve(CalibArgs &a, void *ws);
// synchronises the stream once per Jacobi sweep (the convergence test)
cudaError_t calibrate_launch(const CalibArgs &a, cudaStream_t st);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device the first time a launch needs it (the attribute call is not repeated
// on every launch).
cudaError_t ensure_smem(const void *kernel, int bytes);

// ---------------------------------------------------------------------------
// launchers (return cudaError_t of the launch; shapes already validated)
// ---------------------------------------------------------------------------
// fp32 CUDA-core kernels
cudaError_t simt_encode(const Codec &c, const void *x, int64_t T, uint8_t *ids, uint8_t *codes,
                        void *scales, cudaStream_t st);
cudaError_t simt_attend_dense(int prec, const void *q, int64_t Tq, int H, int d, const void *k,
                              const void *v, int64_t T, float tau, Part out, cudaStream_t st);
cudaError_t simt_attend_full(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                             const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                             Part out, cudaStream_t st);
cudaError_t simt_low_prep(const void *q, int64_t Tq, const Codec &ck, float *qred, float *qc,
                          cudaStream_t st);
cudaError_t simt_attend_low(const float *qred, const float *qc, int64_t Tq, const Codec &ck,
                            const Codec &cv, const Hist &hk, const Hist &hv, int64_t t0,
                            int64_t T, float tau, Part out, cudaStream_t st);
cudaError_t lse_merge_launch(const PartList &parts, int64_t Tq, int H, int d, void *out,
                             int out_prec, float *lse_out, cudaStream_t st);

}  // namespace nanokv
