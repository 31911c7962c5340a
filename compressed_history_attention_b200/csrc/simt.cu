// fp32 CUDA-core kernels for every step of the path.  They serve the fp32
// precision mode (where bf16 tensor cores cannot meet fp32 accuracy) and any
// shape that has no tensor-core kernel.  All arithmetic is fp32.
//
// Method: NanoKV (arXiv 2611.06377) -- Fig. 4(b) encode (nearest center,
// residual projection, INT4 with a per-token scale); Fig. 4(a) full-dim
// decode-attention; Fig. 4(d) low-dim attention with reduced queries and
// output restore, LSE merging.
#include "common.cuh"

#include <math.h>

namespace nanokv {

// ===========================================================================
// encode: one warp per token
// ===========================================================================
template <typename TP, typename TS>
__global__ void __launch_bounds__(256) encode_simt_kernel(const TP *__restrict__ x, int64_t T, int J,
                                                          int r, int C,
                                                          const TP *__restrict__ centers,
                                                          const TP *__restrict__ E,
                                                          uint8_t *__restrict__ ids,
                                                          uint8_t *__restrict__ codes,
                                                          TS *__restrict__ scales) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  float *xs = smem + (size_t)warp * (J + r);
  float *ys = xs + J;
  for (int64_t t = (int64_t)blockIdx.x * wpb + warp; t < T; t += (int64_t)gridDim.x * wpb) {
    const TP *xr = x + t * J;
    for (int i = lane; i < J; i += 32) xs[i] = to_f(xr[i]);
    __syncwarp();
    // nearest center: squared Euclidean distance, strict < keeps the lowest index
    float best = INFINITY;
    int bj = 0;
    for (int j = 0; j < C; ++j) {
      const TP *cr = centers + (size_t)j * J;
      float acc = 0.f;
      for (int i = lane; i < J; i += 32) {
        float df = xs[i] - to_f(cr[i]);
        acc = fmaf(df, df, acc);
      }
      acc = warp_sum(acc);
      if (acc < best) { best = acc; bj = j; }
    }
    // residual and its projection y = E (x - c_a)
    const TP *ca = centers + (size_t)bj * J;
    for (int i = lane; i < J; i += 32) xs[i] -= to_f(ca[i]);
    __syncwarp();
    float m = 0.f;
    for (int k = 0; k < r; ++k) {
      const TP *er = E + (size_t)k * J;
      float acc = 0.f;
      for (int i = lane; i < J; i += 32) acc = fmaf(to_f(er[i]), xs[i], acc);
      acc = warp_sum(acc);
      if (lane == 0) ys[k] = acc;
      m = fmaxf(m, fabsf(acc));
    }
    __syncwarp();
    // per-token symmetric scale in storage precision, INT4 codes in [-7, 7]
    const TS s = from_f<TS>(m / 7.0f);
    const float sf = to_f(s);
    uint8_t *cr = codes + t * (r / 2);
    for (int b = lane; b < r / 2; b += 32) {
      int q0 = 0, q1 = 0;
      if (sf > 0.f) {
        q0 = (int)fminf(7.f, fmaxf(-7.f, rintf(ys[2 * b] / sf)));
        q1 = (int)fminf(7.f, fmaxf(-7.f, rintf(ys[2 * b + 1] / sf)));
      }
      cr[b] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
    }
    if (lane == 0) {
      ids[t] = (uint8_t)bj;
      scales[t] = s;
    }
    __syncwarp();
  }
}

cudaError_t simt_encode(const Codec &c, const void *x, int64_t T, uint8_t *ids, uint8_t *codes,
                        void *scales, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int J = c.H * c.d;
  // warps per block: up to 8, as many as the per-warp token and residual
  // buffers (J + r floats each) leave room for in 227 KB of shared memory;
  // the widest codec (J = 32768, r = 512) runs one warp per block
  const size_t per_warp = (size_t)(J + c.r) * sizeof(float);
  int wpb = (int)(size_t(232448) / per_warp);
  wpb = wpb < 1 ? 1 : (wpb > 8 ? 8 : wpb);
  const size_t smem = (size_t)wpb * per_warp;
  int64_t blocks = (T + wpb - 1) / wpb;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (c.prec == PREC_F32) {
    auto k = encode_simt_kernel<float, float>;
    ensure_smem((const void *)k, (int)smem);
    k<<<(unsigned)blocks, wpb * 32, smem, st>>>((const float *)x, T, J, c.r, c.C,
                                                (const float *)c.centers, (const float *)c.E, ids,
                                                codes, (float *)scales);
  } else {
    auto k = encode_simt_kernel<__nv_bfloat16, __half>;
    ensure_smem((const void *)k, (int)smem);
    k<<<(unsigned)blocks, wpb * 32, smem, st>>>(
        (const __nv_bfloat16 *)x, T, J, c.r, c.C, (const __nv_bfloat16 *)c.centers,
        (const __nv_bfloat16 *)c.E, ids, codes, (__half *)scales);
  }
  return cudaGetLastError();
}

// ===========================================================================
// full-dim decode-attention and dense attention (current chunk)
//   block = 128 threads = 32 query rows x 4 threads; each thread owns d/4
//   output dims.  Key tiles of 32 are produced into shared memory (decoded
//   from codes, or copied), then scored with a per-tile online softmax.
// ===========================================================================
constexpr int SA_BQ = 32, SA_BK = 32, SA_THREADS = 128, SA_TPR = 4;

template <typename TIO, typename TS, int DH, bool DECODE>
__global__ void __launch_bounds__(SA_THREADS)
    attn_simt_kernel(const TIO *__restrict__ q, int64_t Tq, int H,
                     const TIO *__restrict__ kd, const TIO *__restrict__ vd,  // dense [T,H,DH]
                     Codec ck, Codec cv, Hist hk, Hist hv, int64_t t0, int64_t T, float tau,
                     float *__restrict__ Oout, float *__restrict__ Lout) {
  extern __shared__ float sm[];
  float *Ks = sm;                      // [BK][DH]
  float *Vs = Ks + SA_BK * DH;         // [BK][DH]
  int8_t *ck8 = (int8_t *)(Vs + SA_BK * DH);  // [BK][rk]
  int8_t *cv8 = ck8 + SA_BK * (DECODE ? ck.r : 0);

  const int h = blockIdx.y;
  const int tid = threadIdx.x;
  const int row = tid / SA_TPR, sub = tid % SA_TPR;
  constexpr int W = DH / SA_TPR;
  const int64_t qi = (int64_t)blockIdx.x * SA_BQ + row;
  const int J = H * DH;

  float qr[W], o[W];
#pragma unroll
  for (int k = 0; k < W; ++k) {
    qr[k] = qi < Tq ? tau * to_f(q[qi * J + h * DH + sub * W + k]) : 0.f;
    o[k] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  for (int64_t kt = 0; kt < T; kt += SA_BK) {
    const int nk = (int)(T - kt < SA_BK ? T - kt : SA_BK);
    __syncthreads();
    if constexpr (!DECODE) {
      for (int e = tid; e < SA_BK * DH; e += SA_THREADS) {
        const int t = e / DH, i = e % DH;
        float kv = 0.f, vv = 0.f;
        if (t < nk) {
          const int64_t src = (kt + t) * J + h * DH + i;
          kv = to_f(kd[src]);
          vv = to_f(vd[src]);
        }
        Ks[e] = kv;
        Vs[e] = vv;
      }
    } else {
      // unpack this tile's codes (K and V) into int8 shared memory
      const int bk = ck.r / 2, bv = cv.r / 2;
      for (int e = tid; e < SA_BK * bk; e += SA_THREADS) {
        const int t = e / bk, b = e % bk;
        uint8_t by = t < nk ? hk.codes[(t0 + kt + t) * bk + b] : 0;
        ck8[t * ck.r + 2 * b] = (int8_t)nib_lo(by);
        ck8[t * ck.r + 2 * b + 1] = (int8_t)nib_hi(by);
      }
      for (int e = tid; e < SA_BK * bv; e += SA_THREADS) {
        const int t = e / bv, b = e % bv;
        uint8_t by = t < nk ? hv.codes[(t0 + kt + t) * bv + b] : 0;
        cv8[t * cv.r + 2 * b] = (int8_t)nib_lo(by);
        cv8[t * cv.r + 2 * b + 1] = (int8_t)nib_hi(by);
      }
      __syncthreads();
      // decode: X[t][i] = c[a_t][h*DH+i] + s_t * sum_j D[h*DH+i][j] code[t][j]
      constexpr int G = SA_THREADS / DH > 0 ? SA_THREADS / DH : 1;
      constexpr int KPT = SA_BK / G;
      const int i = tid % DH, g = tid / DH;
      if (g < G) {
        const TIO *Dk = (const TIO *)ck.D + (size_t)(h * DH + i) * ck.r;
        const TIO *Dv = (const TIO *)cv.D + (size_t)(h * DH + i) * cv.r;
        float acc[KPT];
#pragma unroll
        for (int u = 0; u < KPT; ++u) acc[u] = 0.f;
        for (int j = 0; j < ck.r; ++j) {
          const float dj = to_f(Dk[j]);
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[u] = fmaf(dj, (float)ck8[(g * KPT + u) * ck.r + j], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < KPT; ++u) {
          const int t = g * KPT + u;
          float val = 0.f;
          if (t < nk) {
            const int64_t tt = t0 + kt + t;
            const float s = to_f(((const TS *)hk.scales)[tt]);
            const int a = min((int)hk.ids[tt], ck.C - 1);
            val = to_f(((const TIO *)ck.centers)[(size_t)a * J + h * DH + i]) + s * acc[u];
          }
          Ks[t * DH + i] = val;
        }
#pragma unroll
        for (int u = 0; u < KPT; ++u) acc[u] = 0.f;
        for (int j = 0; j < cv.r; ++j) {
          const float dj = to_f(Dv[j]);
#pragma unroll
          for (int u = 0; u < KPT; ++u) acc[u] = fmaf(dj, (float)cv8[(g * KPT + u) * cv.r + j], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < KPT; ++u) {
          const int t = g * KPT + u;
          float val = 0.f;
          if (t < nk) {
            const int64_t tt = t0 + kt + t;
            const float s = to_f(((const TS *)hv.scales)[tt]);
            const int a = min((int)hv.ids[tt], cv.C - 1);
            val = to_f(((const TIO *)cv.centers)[(size_t)a * J + h * DH + i]) + s * acc[u];
          }
          Vs[t * DH + i] = val;
        }
      }
    }
    __syncthreads();
    // scores of this tile
    float z[SA_BK];
    float tmax = -INFINITY;
#pragma unroll
    for (int t = 0; t < SA_BK; ++t) {
      float p = 0.f;
#pragma unroll
      for (int k = 0; k < W; ++k) p = fmaf(qr[k], Ks[t * DH + sub * W + k], p);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      z[t] = t < nk ? p : -INFINITY;
      tmax = fmaxf(tmax, z[t]);
    }
    const float mn = fmaxf(m, tmax);
    const float corr = expf(m - mn);  // m = -inf on the first tile -> 0
    l *= corr;
#pragma unroll
    for (int k = 0; k < W; ++k) o[k] *= corr;
#pragma unroll
    for (int t = 0; t < SA_BK; ++t) {
      const float p = expf(z[t] - mn);
      l += p;
#pragma unroll
      for (int k = 0; k < W; ++k) o[k] = fmaf(p, Vs[t * DH + sub * W + k], o[k]);
    }
    m = mn;
  }
  if (qi < Tq) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int k = 0; k < W; ++k) Oout[qi * J + h * DH + sub * W + k] = o[k] * inv;
    if (sub == 0) Lout[(int64_t)h * Tq + qi] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

template <typename TIO, typename TS, int DH, bool DECODE>
static cudaError_t launch_attn_simt(const void *q, int64_t Tq, int H, const void *k, const void *v,
                                    const Codec &ck, const Codec &cv, const Hist &hk,
                                    const Hist &hv, int64_t t0, int64_t T, float tau, Part out,
                                    cudaStream_t st) {
  auto kern = attn_simt_kernel<TIO, TS, DH, DECODE>;
  size_t smem = 2 * SA_BK * DH * sizeof(float);
  if (DECODE) smem += (size_t)SA_BK * (ck.r + cv.r);
  ensure_smem((const void *)kern, (int)smem);
  dim3 grid((unsigned)((Tq + SA_BQ - 1) / SA_BQ), (unsigned)H);
  kern<<<grid, SA_THREADS, smem, st>>>((const TIO *)q, Tq, H, (const TIO *)k, (const TIO *)v, ck,
                                        cv, hk, hv, t0, T, tau, out.O, out.LSE);
  return cudaGetLastError();
}

template <bool DECODE>
static cudaError_t attn_dispatch(int prec, int d, const void *q, int64_t Tq, int H, const void *k,
                                 const void *v, const Codec &ck, const Codec &cv, const Hist &hk,
                                 const Hist &hv, int64_t t0, int64_t T, float tau, Part out,
                                 cudaStream_t st) {
#define NANOKV_ATTN_CASE(DH)                                                                     \
  case DH:                                                                                       \
    return prec == PREC_F32                                                                      \
               ? launch_attn_simt<float, float, DH, DECODE>(q, Tq, H, k, v, ck, cv, hk, hv, t0,  \
                                                            T, tau, out, st)                     \
               : launch_attn_simt<__nv_bfloat16, __half, DH, DECODE>(q, Tq, H, k, v, ck, cv, hk, \
                                                                     hv, t0, T, tau, out, st);
  switch (d) {
    NANOKV_ATTN_CASE(16)
    NANOKV_ATTN_CASE(32)
    NANOKV_ATTN_CASE(64)
    NANOKV_ATTN_CASE(128)
    default:
      return cudaErrorInvalidValue;
  }
#undef NANOKV_ATTN_CASE
}

cudaError_t simt_attend_dense(int prec, const void *q, int64_t Tq, int H, int d, const void *k,
                              const void *v, int64_t T, float tau, Part out, cudaStream_t st) {
  Codec c{};
  Hist hh{};
  return attn_dispatch<false>(prec, d, q, Tq, H, k, v, c, c, hh, hh, 0, T, tau, out, st);
}

cudaError_t simt_attend_full(const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                             const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                             Part out, cudaStream_t st) {
  return attn_dispatch<true>(ck.prec, ck.d, q, Tq, ck.H, nullptr, nullptr, ck, cv, hk, hv, t0, T,
                             tau, out, st);
}

// ===========================================================================
// low-dim prep: q~ = D_{K,h}^T q_h  [H][Tq][r],  qc = C_{K,h} q_h  [H][Tq][C]
// ===========================================================================
template <typename TIO>
__global__ void low_prep_kernel(const TIO *__restrict__ q, int64_t Tq, int H, int d, int r, int C,
                                const TIO *__restrict__ D, const TIO *__restrict__ cen,
                                float *__restrict__ qred, float *__restrict__ qc) {
  extern __shared__ float qs[];  // [16][d]
  const int h = blockIdx.y;
  const int64_t i0 = (int64_t)blockIdx.x * 16;
  const int J = H * d;
  for (int e = threadIdx.x; e < 16 * d; e += blockDim.x) {
    const int64_t i = i0 + e / d;
    qs[e] = i < Tq ? to_f(q[i * J + h * d + e % d]) : 0.f;
  }
  __syncthreads();
  const int per = r + C;
  for (int e = threadIdx.x; e < 16 * per; e += blockDim.x) {
    const int rr = e / per, j = e % per;
    const int64_t i = i0 + rr;
    if (i >= Tq) continue;
    float acc = 0.f;
    if (j < r) {
      for (int k = 0; k < d; ++k) acc = fmaf(qs[rr * d + k], to_f(D[(size_t)(h * d + k) * r + j]), acc);
      qred[((int64_t)h * Tq + i) * r + j] = acc;
    } else {
      const int c = j - r;
      for (int k = 0; k < d; ++k) acc = fmaf(qs[rr * d + k], to_f(cen[(size_t)c * J + h * d + k]), acc);
      qc[((int64_t)h * Tq + i) * C + c] = acc;
    }
  }
}

cudaError_t simt_low_prep(const void *q, int64_t Tq, const Codec &ck, float *qred, float *qc,
                          cudaStream_t st) {
  dim3 grid((unsigned)((Tq + 15) / 16), (unsigned)ck.H);
  const size_t smem = 16 * ck.d * sizeof(float);
  if (ck.prec == PREC_F32)
    low_prep_kernel<float><<<grid, 256, smem, st>>>((const float *)q, Tq, ck.H, ck.d, ck.r, ck.C,
                                                     (const float *)ck.D,
                                                     (const float *)ck.centers, qred, qc);
  else
    low_prep_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(
        (const __nv_bfloat16 *)q, Tq, ck.H, ck.d, ck.r, ck.C, (const __nv_bfloat16 *)ck.D,
        (const __nv_bfloat16 *)ck.centers, qred, qc);
  return cudaGetLastError();
}

// ===========================================================================
// low-dim attention: 16 query rows x 8 threads per block.  Reduced queries,
// accumulators of sum p s code (length rv) and of sum p onehot(a) (length Cv)
// live in shared memory; output restored at the end:
//   O = (sum_c PC[c] c_{V,c,h} + D_{V,h} Oacc) / l
// ===========================================================================
constexpr int SL_BQ = 16, SL_TPR = 8, SL_THREADS = SL_BQ * SL_TPR, SL_BK = 32;

template <typename TIO, typename TS>
__global__ void __launch_bounds__(SL_THREADS)
    attn_low_simt_kernel(const float *__restrict__ qred, const float *__restrict__ qc, int64_t Tq,
                         Codec ck, Codec cv, Hist hk, Hist hv, int64_t t0, int64_t T, float tau,
                         float *__restrict__ Oout, float *__restrict__ Lout) {
  extern __shared__ float sm[];
  const int rk = ck.r, rv = cv.r, Ck = ck.C, Cv = cv.C, d = ck.d, H = ck.H;
  const int J = H * d;
  float *Qs = sm;                         // [BQ][rk]
  float *QCs = Qs + SL_BQ * rk;           // [BQ][Ck]
  float *Oa = QCs + SL_BQ * Ck;           // [BQ][rv]
  float *PC = Oa + SL_BQ * rv;            // [BQ][Cv+1]
  float *sk = PC + SL_BQ * (Cv + 1);      // [BK]
  float *sv = sk + SL_BK;                 // [BK]
  int *ik = (int *)(sv + SL_BK);          // [BK]
  int *iv = ik + SL_BK;                   // [BK]
  int8_t *ck8 = (int8_t *)(iv + SL_BK);   // [BK][rk]
  int8_t *cv8 = ck8 + SL_BK * rk;         // [BK][rv]

  const int h = blockIdx.y;
  const int tid = threadIdx.x, row = tid / SL_TPR, sub = tid % SL_TPR;
  const int64_t qi0 = (int64_t)blockIdx.x * SL_BQ;
  const int64_t qi = qi0 + row;

  for (int e = tid; e < SL_BQ * rk; e += SL_THREADS) {
    const int64_t i = qi0 + e / rk;
    Qs[e] = i < Tq ? qred[((int64_t)h * Tq + i) * rk + e % rk] : 0.f;
  }
  for (int e = tid; e < SL_BQ * Ck; e += SL_THREADS) {
    const int64_t i = qi0 + e / Ck;
    QCs[e] = i < Tq ? qc[((int64_t)h * Tq + i) * Ck + e % Ck] : 0.f;
  }
  for (int e = tid; e < SL_BQ * rv; e += SL_THREADS) Oa[e] = 0.f;
  for (int e = tid; e < SL_BQ * (Cv + 1); e += SL_THREADS) PC[e] = 0.f;

  float m = -INFINITY, l = 0.f;
  for (int64_t kt = 0; kt < T; kt += SL_BK) {
    const int nk = (int)(T - kt < SL_BK ? T - kt : SL_BK);
    __syncthreads();
    for (int e = tid; e < SL_BK * (rk / 2); e += SL_THREADS) {
      const int t = e / (rk / 2), b = e % (rk / 2);
      uint8_t by = t < nk ? hk.codes[(t0 + kt + t) * (rk / 2) + b] : 0;
      ck8[t * rk + 2 * b] = (int8_t)nib_lo(by);
      ck8[t * rk + 2 * b + 1] = (int8_t)nib_hi(by);
    }
    for (int e = tid; e < SL_BK * (rv / 2); e += SL_THREADS) {
      const int t = e / (rv / 2), b = e % (rv / 2);
      uint8_t by = t < nk ? hv.codes[(t0 + kt + t) * (rv / 2) + b] : 0;
      cv8[t * rv + 2 * b] = (int8_t)nib_lo(by);
      cv8[t * rv + 2 * b + 1] = (int8_t)nib_hi(by);
    }
    for (int t = tid; t < SL_BK; t += SL_THREADS) {
      const bool ok = t < nk;
      const int64_t tt = t0 + kt + t;
      sk[t] = ok ? to_f(((const TS *)hk.scales)[tt]) : 0.f;
      sv[t] = ok ? to_f(((const TS *)hv.scales)[tt]) : 0.f;
      ik[t] = ok ? min((int)hk.ids[tt], Ck - 1) : 0;
      iv[t] = ok ? min((int)hv.ids[tt], Cv - 1) : 0;
    }
    __syncthreads();
    float z[SL_BK];
    float tmax = -INFINITY;
    for (int t = 0; t < SL_BK; ++t) {
      float p = 0.f;
      for (int j = sub; j < rk; j += SL_TPR) p = fmaf(Qs[row * rk + j], (float)ck8[t * rk + j], p);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      p += __shfl_xor_sync(0xffffffffu, p, 4);
      const float zz = tau * (sk[t] * p + QCs[row * Ck + ik[t]]);
      z[t] = t < nk ? zz : -INFINITY;
      tmax = fmaxf(tmax, z[t]);
    }
    const float mn = fmaxf(m, tmax);
    const float corr = expf(m - mn);
    l *= corr;
    for (int j = sub; j < rv; j += SL_TPR) Oa[row * rv + j] *= corr;
    for (int c = sub; c < Cv; c += SL_TPR) PC[row * (Cv + 1) + c] *= corr;
    __syncwarp();
    for (int t = 0; t < SL_BK; ++t) {
      const float p = expf(z[t] - mn);
      l += p;
      const float ps = p * sv[t];
      for (int j = sub; j < rv; j += SL_TPR) Oa[row * rv + j] = fmaf(ps, (float)cv8[t * rv + j], Oa[row * rv + j]);
      if (sub == 0 && t < nk) PC[row * (Cv + 1) + iv[t]] += p;
      __syncwarp();
    }
    m = mn;
  }
  __syncthreads();
  if (qi < Tq) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const TIO *Dv = (const TIO *)cv.D;
    const TIO *Cen = (const TIO *)cv.centers;
    for (int k = sub; k < d; k += SL_TPR) {
      float acc = 0.f;
      for (int c = 0; c < Cv; ++c) acc = fmaf(PC[row * (Cv + 1) + c], to_f(Cen[(size_t)c * J + h * d + k]), acc);
      for (int j = 0; j < rv; ++j) acc = fmaf(Oa[row * rv + j], to_f(Dv[(size_t)(h * d + k) * rv + j]), acc);
      Oout[qi * J + h * d + k] = acc * inv;
    }
    if (sub == 0) Lout[(int64_t)h * Tq + qi] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

cudaError_t simt_attend_low(const float *qred, const float *qc, int64_t Tq, const Codec &ck,
                            const Codec &cv, const Hist &hk, const Hist &hv, int64_t t0,
                            int64_t T, float tau, Part out, cudaStream_t st) {
  const size_t smem = sizeof(float) * (SL_BQ * (ck.r + ck.C + cv.r + cv.C + 1) + 2 * SL_BK) +
                      sizeof(int) * 2 * SL_BK + (size_t)SL_BK * (ck.r + cv.r);
  dim3 grid((unsigned)((Tq + SL_BQ - 1) / SL_BQ), (unsigned)ck.H);
  if (ck.prec == PREC_F32) {
    auto k = attn_low_simt_kernel<float, float>;
    ensure_smem((const void *)k, (int)smem);
    k<<<grid, SL_THREADS, smem, st>>>(qred, qc, Tq, ck, cv, hk, hv, t0, T, tau, out.O, out.LSE);
  } else {
    auto k = attn_low_simt_kernel<__nv_bfloat16, __half>;
    ensure_smem((const void *)k, (int)smem);
    k<<<grid, SL_THREADS, smem, st>>>(qred, qc, Tq, ck, cv, hk, hv, t0, T, tau, out.O, out.LSE);
  }
  return cudaGetLastError();
}

// ===========================================================================
// LSE merge: one thread per 4 output elements (d is a multiple of 4)
// ===========================================================================
template <typename TO>
__global__ void lse_merge_kernel(PartList parts, int64_t Tq, int H, int d, TO *__restrict__ out,
                                 float *__restrict__ lse_out) {
  const int64_t n4 = Tq * H * d / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t idx = e * 4;
    const int64_t i = idx / ((int64_t)H * d);
    const int h = (int)((idx / d) % H);
    const int k = (int)(idx % d);
    float lse[kMaxParts];
    float m = -INFINITY;
    for (int b = 0; b < parts.n; ++b) {
      lse[b] = parts.LSE[b][(int64_t)h * Tq + i];
      m = fmaxf(m, lse[b]);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = -INFINITY;
    if (m > -INFINITY) {
      float tot = 0.f;
      for (int b = 0; b < parts.n; ++b) tot += expf(lse[b] - m);
      const float inv = 1.f / tot;
      for (int b = 0; b < parts.n; ++b) {
        const float w = expf(lse[b] - m) * inv;
        if (w == 0.f) continue;
        const float4 o = *(const float4 *)(parts.O[b] + idx);
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
      }
      L = m + logf(tot);
    }
    out[idx] = from_f<TO>(acc.x);
    out[idx + 1] = from_f<TO>(acc.y);
    out[idx + 2] = from_f<TO>(acc.z);
    out[idx + 3] = from_f<TO>(acc.w);
    if (lse_out && k == 0) lse_out[(int64_t)h * Tq + i] = L;
  }
}

cudaError_t lse_merge_launch(const PartList &parts, int64_t Tq, int H, int d, void *out,
                             int out_prec, float *lse_out, cudaStream_t st) {
  const int64_t n4 = Tq * H * d / 4;
  if (n4 == 0) return cudaSuccess;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (out_prec == PREC_F32)
    lse_merge_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(parts, Tq, H, d, (float *)out, lse_out);
  else
    lse_merge_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(parts, Tq, H, d,
                                                                    (__nv_bfloat16 *)out, lse_out);
  return cudaGetLastError();
}

}  // namespace nanokv
