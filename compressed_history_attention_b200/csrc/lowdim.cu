// Reduced attention dimension per head (NanoKV-Fast: Table 6, head-layer
// pairs deployed at d_h in {32, 64, 96, 128}; Fig. 4(d), the low-dimensional
// branch reduces the queries and restores the output dimension; Table 8,
// low-dimensional maps).  Head h attends through orthonormal maps U_h
// (queries, keys) and W_h (values, output restore), [d, d_h] each, stored
// padded as [H, d, d] with head h's map in columns [0, d_h).
//
// The stored coefficients are reused: a key decodes straight into d_h
// dimensions, k~ = U_h^T c_K[a] + s (U_h^T D_K,h) code, so the decoder rows
// and centers are mapped once per codec (lowdim_prepare) and the full-dim
// decode-attention kernel runs on them at width d_h.  Only the leading d_h
// columns of a map matter for a head at d_h, so the tables hold all d
// mapped rows and serve every d_h.
#include "common.cuh"

namespace nanokv {

namespace {

constexpr int kD = 128;

// out rows [h*128 + j] of the mapped decoder: sum_i M[h][i][j] D[h*128 + i][k]
// (blockIdx.x: 256 consecutive (j, k) outputs of one head, blockIdx.y: head);
// mapped centers: out[a][h*128 + j] = sum_i c[a][h*128 + i] M[h][i][j].
__global__ void __launch_bounds__(256) mapped_decoder_kernel(const __nv_bfloat16 *__restrict__ D,
                                                             const __nv_bfloat16 *__restrict__ M, int r,
                                                             __nv_bfloat16 *__restrict__ out) {
  const int h = blockIdx.y;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // j * r + k
  if (idx >= (int64_t)kD * r) return;
  const int j = (int)(idx / r), k = (int)(idx % r);
  const __nv_bfloat16 *Mh = M + (size_t)h * kD * kD;
  const __nv_bfloat16 *Dh = D + (size_t)h * kD * r;
  float acc = 0.f;
#pragma unroll 8
  for (int i = 0; i < kD; ++i) acc = fmaf(__bfloat162float(Mh[i * kD + j]), __bfloat162float(Dh[(size_t)i * r + k]), acc);
  out[((size_t)h * kD + j) * r + k] = __float2bfloat16_rn(acc);
}

__global__ void __launch_bounds__(128) mapped_centers_kernel(const __nv_bfloat16 *__restrict__ cen,
                                                             const __nv_bfloat16 *__restrict__ M, int H,
                                                             __nv_bfloat16 *__restrict__ out) {
  const int a = blockIdx.x, h = blockIdx.y, j = threadIdx.x;
  const int J = H * kD;
  const __nv_bfloat16 *Mh = M + (size_t)h * kD * kD;
  const __nv_bfloat16 *c = cen + (size_t)a * J + (size_t)h * kD;
  float acc = 0.f;
#pragma unroll 8
  for (int i = 0; i < kD; ++i) acc = fmaf(__bfloat162float(c[i]), __bfloat162float(Mh[i * kD + j]), acc);
  out[(size_t)a * J + (size_t)h * kD + j] = __float2bfloat16_rn(acc);
}

// Reduced queries q~ = U_h^T q for the listed heads: [Tq, H*128] bf16, head
// h's d_h values in columns [h*128, h*128 + d_h), zeros after them.  Block:
// 128 threads (output column j), kQRows query rows, one head; each thread
// keeps its map column in registers, the rows are staged in shared memory.
constexpr int kQRows = 32;

__global__ void __launch_bounds__(128) reduce_queries_kernel(const __nv_bfloat16 *__restrict__ q, int64_t Tq, int H,
                                                             const __nv_bfloat16 *__restrict__ U,
                                                             const int32_t *__restrict__ heads, const HeadDims dims,
                                                             __nv_bfloat16 *__restrict__ qred) {
  __shared__ float sq[kQRows][kD];
  const int h = heads[blockIdx.y];
  const int dh = dims.d[h];
  const int j = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * kQRows;
  for (int e = threadIdx.x; e < kQRows * kD; e += 128) {
    const int64_t t = t0 + e / kD;
    sq[e / kD][e % kD] = t < Tq ? __bfloat162float(q[(t * H + h) * kD + e % kD]) : 0.f;
  }
  float u[kD];
  const __nv_bfloat16 *Uh = U + (size_t)h * kD * kD;
#pragma unroll
  for (int i = 0; i < kD; ++i) u[i] = j < dh ? __bfloat162float(Uh[i * kD + j]) : 0.f;
  __syncthreads();
  for (int rr = 0; rr < kQRows; ++rr) {
    const int64_t t = t0 + rr;
    if (t >= Tq) break;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kD; ++i) acc = fmaf(u[i], sq[rr][i], acc);
    qred[t * H * kD + (int64_t)h * kD + j] = __float2bfloat16_rn(acc);
  }
}

// Analytical maps (Table 8, "analytical initialization"): per head, the
// left singular vectors of the decoder rows D_h [128, r], ordered by
// decreasing singular value, as the eigenvectors of G = D_h D_h^T.  One CTA
// per head runs cyclic Jacobi on G in shared memory (Golub and Van Loan,
// "Matrix Computations", the symmetric Schur decomposition by Jacobi
// rotations, with the round-robin ordering that lets a round rotate 64
// disjoint index pairs at once).  Sweeps stop when the off-diagonal mass is
// below 1e-6 of the total (Frobenius norms), or after kJacobiSweeps.
constexpr int kJacobiSweeps = 20;
constexpr int kLd = kD + 1;  // padded row: column accesses hit distinct banks

__global__ void __launch_bounds__(512) analytic_maps_kernel(const __nv_bfloat16 *__restrict__ D, int r,
                                                            __nv_bfloat16 *__restrict__ maps) {
  extern __shared__ float jsm[];
  float *A = jsm;               // [128][kLd]
  float *V = A + kD * kLd;      // [128][kLd]
  __shared__ float cs[64], sn[64];
  __shared__ int pp[64], qq[64];
  __shared__ float red[2][16];
  __shared__ int done;
  const int h = blockIdx.x, tid = threadIdx.x;
  const __nv_bfloat16 *Dh = D + (size_t)h * kD * r;
  // G = D_h D_h^T (fp32 sums of bf16 products), V = I
  for (int e = tid; e < kD * kD; e += 512) {
    const int i = e / kD, j = e % kD;
    float acc = 0.f;
    if (j >= i) {
      const __nv_bfloat16 *a = Dh + (size_t)i * r, *b = Dh + (size_t)j * r;
      for (int k = 0; k < r; ++k) acc = fmaf(__bfloat162float(a[k]), __bfloat162float(b[k]), acc);
    }
    A[i * kLd + j] = acc;
    V[i * kLd + j] = i == j ? 1.f : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < kD * kD; e += 512) {
    const int i = e / kD, j = e % kD;
    if (j < i) A[i * kLd + j] = A[j * kLd + i];
  }
  if (tid == 0) done = 0;
  __syncthreads();
  for (int sweep = 0; sweep < kJacobiSweeps && !done; ++sweep) {
    for (int k = 0; k < kD - 1; ++k) {
      // round k of the circle schedule: (127, k) and ((k + i) % 127, (k - i) % 127)
      if (tid < 64) {
        const int i = tid;
        int p = i == 0 ? kD - 1 : (k + i) % (kD - 1);
        int q = i == 0 ? k : (k - i + (kD - 1)) % (kD - 1);
        if (p > q) { const int t = p; p = q; q = t; }
        const float apq = A[p * kLd + q], app = A[p * kLd + p], aqq = A[q * kLd + q];
        float c = 1.f, s = 0.f;
        if (fabsf(apq) > 1e-30f) {
          const float tau = (aqq - app) / (2.f * apq);
          const float t = (tau >= 0.f ? 1.f : -1.f) / (fabsf(tau) + sqrtf(1.f + tau * tau));
          c = rsqrtf(1.f + t * t);
          s = t * c;
        }
        cs[i] = c;
        sn[i] = s;
        pp[i] = p;
        qq[i] = q;
      }
      __syncthreads();
      // columns: A <- A J and V <- V J
      for (int e = tid; e < 64 * kD; e += 512) {
        const int i = e / kD, row = e % kD;
        const int p = pp[i], q = qq[i];
        const float c = cs[i], s = sn[i];
        const float ap = A[row * kLd + p], aq = A[row * kLd + q];
        A[row * kLd + p] = c * ap - s * aq;
        A[row * kLd + q] = s * ap + c * aq;
        const float vp = V[row * kLd + p], vq = V[row * kLd + q];
        V[row * kLd + p] = c * vp - s * vq;
        V[row * kLd + q] = s * vp + c * vq;
      }
      __syncthreads();
      // rows: A <- J^T A
      for (int e = tid; e < 64 * kD; e += 512) {
        const int i = e / kD, col = e % kD;
        const int p = pp[i], q = qq[i];
        const float c = cs[i], s = sn[i];
        const float ap = A[p * kLd + col], aq = A[q * kLd + col];
        A[p * kLd + col] = c * ap - s * aq;
        A[q * kLd + col] = s * ap + c * aq;
      }
      __syncthreads();
    }
    // convergence: off-diagonal against total squared mass
    float off = 0.f, tot = 0.f;
    for (int e = tid; e < kD * kD; e += 512) {
      const float v = A[(e / kD) * kLd + e % kD];
      tot += v * v;
      if (e / kD != e % kD) off += v * v;
    }
    off = warp_sum(off);
    tot = warp_sum(tot);
    if ((tid & 31) == 0) {
      red[0][tid >> 5] = off;
      red[1][tid >> 5] = tot;
    }
    __syncthreads();
    if (tid == 0) {
      float o = 0.f, t = 0.f;
      for (int w = 0; w < 16; ++w) {
        o += red[0][w];
        t += red[1][w];
      }
      done = !(o > 1e-12f * t);
    }
    __syncthreads();
  }
  // order by decreasing eigenvalue (ties by index) and write the columns
  if (tid < kD) {
    const float ev = A[tid * kLd + tid];
    int rank = 0;
    for (int j = 0; j < kD; ++j) {
      const float o = A[j * kLd + j];
      rank += (o > ev) || (o == ev && j < tid);
    }
    for (int row = 0; row < kD; ++row)
      maps[(size_t)h * kD * kD + (size_t)row * kD + rank] = __float2bfloat16_rn(V[row * kLd + tid]);
  }
}

}  // namespace

cudaError_t lowdim_analytic(const Codec &c, void *maps, cudaStream_t st) {
  const int smem = 2 * kD * kLd * (int)sizeof(float);
  cudaError_t e = ensure_smem((const void *)analytic_maps_kernel, smem);
  if (e != cudaSuccess) return e;
  analytic_maps_kernel<<<(unsigned)c.H, 512, smem, st>>>((const __nv_bfloat16 *)c.D, c.r, (__nv_bfloat16 *)maps);
  return cudaGetLastError();
}

size_t lowdim_aux_bytes(const Codec &ck, const Codec &cv) {
  const size_t J = (size_t)ck.H * kD;
  const size_t dec = J * ck.r * 2;
  return ((2 * dec + ((size_t)ck.C + cv.C) * J * 2) + 255) & ~(size_t)255;
}

LowdimTables lowdim_tables(const Codec &ck, const Codec &cv, void *aux) {
  const size_t J = (size_t)ck.H * kD;
  char *p = (char *)aux;
  LowdimTables t;
  t.D[0] = p;
  t.D[1] = p + J * ck.r * 2;
  t.cen[0] = p + 2 * J * ck.r * 2;
  t.cen[1] = p + 2 * J * ck.r * 2 + (size_t)ck.C * J * 2;
  return t;
}

cudaError_t lowdim_prepare(const Codec &ck, const Codec &cv, const void *U, const void *W, void *aux,
                           cudaStream_t st) {
  const LowdimTables t = lowdim_tables(ck, cv, aux);
  const void *maps[2] = {U, W};
  const Codec *c[2] = {&ck, &cv};
  for (int br = 0; br < 2; ++br) {
    const unsigned nb = (unsigned)(((int64_t)kD * c[br]->r + 255) / 256);
    mapped_decoder_kernel<<<dim3(nb, (unsigned)ck.H), 256, 0, st>>>(
        (const __nv_bfloat16 *)c[br]->D, (const __nv_bfloat16 *)maps[br], c[br]->r, (__nv_bfloat16 *)t.D[br]);
    mapped_centers_kernel<<<dim3((unsigned)c[br]->C, (unsigned)ck.H), 128, 0, st>>>(
        (const __nv_bfloat16 *)c[br]->centers, (const __nv_bfloat16 *)maps[br], ck.H, (__nv_bfloat16 *)t.cen[br]);
  }
  return cudaGetLastError();
}

cudaError_t reduce_queries(const void *q, int64_t Tq, int H, const void *U, HeadSel heads, const HeadDims &dims,
                           void *qred, cudaStream_t st) {
  if (Tq == 0 || heads.n == 0) return cudaSuccess;
  const dim3 grid((unsigned)((Tq + kQRows - 1) / kQRows), (unsigned)heads.n);
  reduce_queries_kernel<<<grid, 128, 0, st>>>((const __nv_bfloat16 *)q, Tq, H, (const __nv_bfloat16 *)U, heads.map,
                                              dims, (__nv_bfloat16 *)qred);
  return cudaGetLastError();
}

}  // namespace nanokv
