// Calibration of one branch's codec on a chunk of tokens, the step before
// encode (NanoKV: Table 5, centers fitted separately for K and V; Table 2,
// joint PCA with INT4 coefficients and shared centers; Fig. 3(a), joint
// head-channel PCA retains the most KV variance at matched compression).
//
//   centers: Lloyd k-means rounds from caller-given initial centers: assign
//            each token to its nearest center (ties to the lowest index),
//            move each center to the mean of its tokens (a center without
//            tokens stays);
//   D:       the r leading eigenvectors of the residual second moment
//            S = (1/N) sum_t (x_t - c_{a_t}) (x_t - c_{a_t})^T over the joint
//            H*d channels, each with its largest-magnitude entry positive;
//            E = D^T.
//
// k-means runs in fp32.  The second moment is accumulated in fp64, and its
// eigenvectors come from cyclic Jacobi in fp64 on S held in global memory
// (Golub and Van Loan, "Matrix Computations": the symmetric Schur
// decomposition by Jacobi rotations, round-robin ordering so that one round
// rotates J/2 disjoint pairs): each round is three launches (rotation
// angles, column rotations of S and of the eigenvector matrix, row rotations
// of S), the kernel boundaries ordering them.  fp64 because the rounding of
// ~2 J rotations per entry and sweep, spread over J^2 entries, grows like
// sqrt(J) * sqrt(2 J sweeps) * eps: about 4e-4 of the largest eigenvalue at
// J = 1536 in fp32, more than the gaps between the leading eigenvalues.
#include "common.cuh"

namespace nanokv {

namespace {

constexpr int kMaxPerLane = 96;  // J <= 3072

template <typename T>
__global__ void __launch_bounds__(256) kmeans_assign_kernel(const T *__restrict__ x, int64_t N, int J,
                                                            const float *__restrict__ cen, int C,
                                                            uint8_t *__restrict__ ids) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= N) return;
  const int per = J / 32;
  float xv[kMaxPerLane];
#pragma unroll
  for (int k = 0; k < kMaxPerLane; ++k)
    if (k < per) xv[k] = to_f(x[t * J + k * 32 + lane]);
  float best = INFINITY;
  int arg = 0;
  for (int j = 0; j < C; ++j) {
    const float *c = cen + (size_t)j * J;
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k)
      if (k < per) {
        const float dlt = xv[k] - c[k * 32 + lane];
        acc = fmaf(dlt, dlt, acc);
      }
    acc = warp_sum(acc);
    if (acc < best) {  // strict: the lowest index wins a tie
      best = acc;
      arg = j;
    }
  }
  if (lane == 0) ids[t] = (uint8_t)arg;
}

// centers[j][col] = mean of the tokens assigned to j (in token order); a
// center without tokens keeps its value.  grid (C, ceil(J / 256)).
template <typename T>
__global__ void __launch_bounds__(256) kmeans_update_kernel(const T *__restrict__ x, int64_t N, int J,
                                                            const uint8_t *__restrict__ ids,
                                                            float *__restrict__ cen) {
  const int j = blockIdx.x;
  const int col = blockIdx.y * 256 + threadIdx.x;
  float acc = 0.f;
  int64_t n = 0;
  for (int64_t t = 0; t < N; ++t)
    if (ids[t] == j) {
      if (col < J) acc += to_f(x[t * J + col]);
      ++n;
    }
  if (col < J && n > 0) cen[(size_t)j * J + col] = acc / (float)n;
}

// S = (1/N) rho^T rho, rho_t = x_t - c_{a_t}: 64 x 64 tiles of the upper
// triangle (mirrored), 32 tokens per step, 4 x 4 outputs per thread.
constexpr int kGT = 64, kGK = 32;

template <typename T>
__global__ void __launch_bounds__(256) residual_gram_kernel(const T *__restrict__ x, int64_t N, int J,
                                                            const float *__restrict__ cen,
                                                            const uint8_t *__restrict__ ids,
                                                            double *__restrict__ S) {
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj < bi) return;
  __shared__ double a[kGK][kGT + 2], b[kGK][kGT + 2];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int i0 = bi * kGT, j0 = bj * kGT;
  double acc[4][4] = {};
  for (int64_t t0 = 0; t0 < N; t0 += kGK) {
    for (int e = threadIdx.x; e < kGK * kGT; e += 256) {
      const int tt = e / kGT, cc = e % kGT;
      const int64_t t = t0 + tt;
      double va = 0.0, vb = 0.0;
      if (t < N) {
        const float *c = cen + (size_t)ids[t] * J;
        if (i0 + cc < J) va = (double)to_f(x[t * J + i0 + cc]) - (double)c[i0 + cc];
        if (j0 + cc < J) vb = (double)to_f(x[t * J + j0 + cc]) - (double)c[j0 + cc];
      }
      a[tt][cc] = va;
      b[tt][cc] = vb;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < kGK; ++k) {
      double ra[4], rb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        ra[u] = a[k][ty * 4 + u];
        rb[u] = b[k][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(ra[u], rb[v], acc[u][v]);
    }
    __syncthreads();
  }
  const double inv = 1.0 / (double)N;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = i0 + ty * 4 + u, j = j0 + tx * 4 + v;
      if (i < J && j < J) {
        S[(size_t)i * J + j] = acc[u][v] * inv;
        S[(size_t)j * J + i] = acc[u][v] * inv;
      }
    }
}

__global__ void identity_kernel(double *__restrict__ V, int n) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < (int64_t)n * n) V[e] = (e / n == e % n) ? 1.0 : 0.0;
}

struct Rot {
  double c, s;
  int p, q;
};

// round k of the circle schedule over n (even) indices: pair 0 is
// (n-1, k), pair i >= 1 is ((k + i) mod (n-1), (k - i) mod (n-1)); p < q.
__global__ void jacobi_angles_kernel(const double *__restrict__ A, int n, int k, Rot *__restrict__ rot,
                                     const int *__restrict__ done) {
  if (*done) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n / 2) return;
  const int m = n - 1;
  int p = i == 0 ? m : (k + i) % m;
  int q = i == 0 ? k : (k - i + m) % m;
  if (p > q) {
    const int t = p;
    p = q;
    q = t;
  }
  const double apq = A[(size_t)p * n + q], app = A[(size_t)p * n + p], aqq = A[(size_t)q * n + q];
  double c = 1.0, s = 0.0;
  if (fabs(apq) > 1e-300) {
    const double tau = (aqq - app) / (2.0 * apq);
    // |tau| large: t ~ 1 / (2 tau), computed without squaring tau
    const double at = fabs(tau);
    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (at + (at > 1e150 ? at : sqrt(1.0 + tau * tau)));
    c = 1.0 / sqrt(1.0 + t * t);
    s = t * c;
  }
  rot[i] = Rot{c, s, p, q};
}

// A <- A J and V <- V J: thread = (row, pair); consecutive threads take
// consecutive pairs of one row.
__global__ void __launch_bounds__(256) jacobi_cols_kernel(double *__restrict__ A, double *__restrict__ V, int n,
                                                          const Rot *__restrict__ rot, const int *__restrict__ done) {
  if (*done) return;
  const int half = n / 2;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)n * half) return;
  const int row = (int)(e / half), i = (int)(e % half);
  const Rot r = rot[i];
  double *a = A + (size_t)row * n, *v = V + (size_t)row * n;
  const double ap = a[r.p], aq = a[r.q];
  a[r.p] = r.c * ap - r.s * aq;
  a[r.q] = r.s * ap + r.c * aq;
  const double vp = v[r.p], vq = v[r.q];
  v[r.p] = r.c * vp - r.s * vq;
  v[r.q] = r.s * vp + r.c * vq;
}

// A <- J^T A: thread = (pair, column).
__global__ void __launch_bounds__(256) jacobi_rows_kernel(double *__restrict__ A, int n, const Rot *__restrict__ rot,
                                                          const int *__restrict__ done) {
  if (*done) return;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)(n / 2) * n) return;
  const int i = (int)(e / n), col = (int)(e % n);
  const Rot r = rot[i];
  double *ap = A + (size_t)r.p * n + col, *aq = A + (size_t)r.q * n + col;
  const double x = *ap, y = *aq;
  *ap = r.c * x - r.s * y;
  *aq = r.s * x + r.c * y;
}

// off-diagonal and total squared mass (offtot[0], offtot[1]); done = off <=
// 1e-20 total (one block)
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(1024) jacobi_check_kernel(const double *__restrict__ A, int n, int *__restrict__ done,
                                                            double *__restrict__ offtot) {
  __shared__ double so[32], st[32];
  double off = 0.0, tot = 0.0;
  for (int64_t e = threadIdx.x; e < (int64_t)n * n; e += 1024) {
    const double v = A[e];
    tot += v * v;
    if (e / n != e % n) off += v * v;
  }
  off = warp_sum_d(off);
  tot = warp_sum_d(tot);
  if ((threadIdx.x & 31) == 0) {
    so[threadIdx.x >> 5] = off;
    st[threadIdx.x >> 5] = tot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double o = 0.0, t = 0.0;
    for (int w = 0; w < 32; ++w) {
      o += so[w];
      t += st[w];
    }
    *done = !(o > 1e-20 * t);
    offtot[0] = o;
    offtot[1] = t;
  }
}

// The r leading eigenvectors: one block per index i; the block of an index
// whose rank (decreasing eigenvalue, ties by index) is below r writes that
// column of D [J, r] and row of E [r, J] with the sign rule, and its
// eigenvalue.
template <typename T>
__global__ void __launch_bounds__(256) select_kernel(const double *__restrict__ A, const double *__restrict__ V, int n,
                                                     int r, T *__restrict__ D, T *__restrict__ E,
                                                     float *__restrict__ evals) {
  const int i = blockIdx.x;
  const double ev = A[(size_t)i * n + i];
  __shared__ int rank_s;
  __shared__ double bm[8];
  __shared__ int bk[8];
  int rk = 0;
  for (int j = threadIdx.x; j < n; j += 256) {
    const double o = A[(size_t)j * n + j];
    rk += (o > ev) || (o == ev && j < i);
  }
  for (int o = 16; o > 0; o >>= 1) rk += __shfl_xor_sync(0xffffffffu, rk, o);
  if (threadIdx.x == 0) rank_s = 0;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) atomicAdd(&rank_s, rk);
  __syncthreads();
  const int rank = rank_s;
  if (rank >= r) return;
  // largest |entry| (first on a tie) of column i of V
  double m = -1.0;
  int mk = 0;
  for (int row = threadIdx.x; row < n; row += 256) {
    const double a = fabs(V[(size_t)row * n + i]);
    if (a > m) {
      m = a;
      mk = row;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const double m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const int k2 = __shfl_xor_sync(0xffffffffu, mk, o);
    if (m2 > m || (m2 == m && k2 < mk)) {
      m = m2;
      mk = k2;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    bm[threadIdx.x >> 5] = m;
    bk[threadIdx.x >> 5] = mk;
  }
  __syncthreads();
  double best = bm[0];
  int bestk = bk[0];
  for (int w = 1; w < 8; ++w)
    if (bm[w] > best || (bm[w] == best && bk[w] < bestk)) {
      best = bm[w];
      bestk = bk[w];
    }
  const double sg = V[(size_t)bestk * n + i] < 0.0 ? -1.0 : 1.0;
  for (int row = threadIdx.x; row < n; row += 256) {
    const T v = from_f<T>((float)(sg * V[(size_t)row * n + i]));
    D[(size_t)row * r + rank] = v;
    E[(size_t)rank * n + row] = v;
  }
  if (threadIdx.x == 0 && evals) evals[rank] = (float)ev;
}

template <typename T>
__global__ void to_param_kernel(const float *__restrict__ src, T *__restrict__ dst, int64_t n) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n) dst[e] = from_f<T>(src[e]);
}

unsigned nblk(int64_t n, int b) { return (unsigned)((n + b - 1) / b); }

template <typename T>
cudaError_t calibrate_t(const CalibArgs &a, cudaStream_t st) {
  const int J = a.J;
  const T *x = (const T *)a.x;
  float *cen = a.cen32;
  cudaError_t e = cudaMemcpyAsync(cen, a.init, (size_t)a.C * J * sizeof(float), cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  const unsigned ga = nblk(a.N, 8);
  const dim3 gu((unsigned)a.C, nblk(J, 256));
  for (int it = 0; it < a.rounds; ++it) {
    kmeans_assign_kernel<T><<<ga, 256, 0, st>>>(x, a.N, J, cen, a.C, a.ids);
    kmeans_update_kernel<T><<<gu, 256, 0, st>>>(x, a.N, J, a.ids, cen);
  }
  kmeans_assign_kernel<T><<<ga, 256, 0, st>>>(x, a.N, J, cen, a.C, a.ids);
  const unsigned nt = nblk(J, kGT);
  residual_gram_kernel<T><<<dim3(nt, nt), 256, 0, st>>>(x, a.N, J, cen, a.ids, a.S);
  identity_kernel<<<nblk((int64_t)J * J, 256), 256, 0, st>>>(a.V, J);
  if ((e = cudaMemsetAsync(a.done, 0, sizeof(int), st)) != cudaSuccess) return e;
  const unsigned gcol = nblk((int64_t)J * (J / 2), 256);
  // sweeps until the off-diagonal mass is below 1e-20 of the total, or has
  // stopped falling (fp32 rounding level: a sweep takes off less than 10%).
  // Early sweeps can shrink it slowly, so only a sweep that makes no
  // progress ends the loop before the threshold.
  double prev_off = INFINITY;
  for (int sweep = 0; sweep < kCalibSweeps; ++sweep) {
    for (int k = 0; k < J - 1; ++k) {
      jacobi_angles_kernel<<<nblk(J / 2, 128), 128, 0, st>>>(a.S, J, k, (Rot *)a.rot, a.done);
      jacobi_cols_kernel<<<gcol, 256, 0, st>>>(a.S, a.V, J, (const Rot *)a.rot, a.done);
      jacobi_rows_kernel<<<gcol, 256, 0, st>>>(a.S, J, (const Rot *)a.rot, a.done);
    }
    jacobi_check_kernel<<<1, 1024, 0, st>>>(a.S, J, a.done, (double *)(a.done + 4));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int h_done = 0;
    double ot[2] = {0.0, 0.0};
    if ((e = cudaMemcpyAsync(&h_done, a.done, sizeof(int), cudaMemcpyDeviceToHost, st)) != cudaSuccess) return e;
    if ((e = cudaMemcpyAsync(ot, a.done + 4, sizeof(ot), cudaMemcpyDeviceToHost, st)) != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
    if (h_done || ot[0] > 0.9 * prev_off) break;
    prev_off = ot[0];
  }
  select_kernel<T><<<(unsigned)J, 256, 0, st>>>(a.S, a.V, J, a.r, (T *)a.D, (T *)a.E, a.evals);
  to_param_kernel<T><<<nblk((int64_t)a.C * J, 256), 256, 0, st>>>(cen, (T *)a.centers, (int64_t)a.C * J);
  return cudaGetLastError();
}

}  // namespace

size_t calibrate_workspace(int64_t N, int J, int C) {
  auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
  return al((size_t)C * J * 4) + 2 * al((size_t)J * J * 8) + al((size_t)(J / 2) * sizeof(Rot)) + al(sizeof(int)) +
         al((size_t)N);
}

void calibrate_carve(CalibArgs &a, void *ws) {
  auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
  char *p = (char *)ws;
  a.cen32 = (float *)p;
  p += al((size_t)a.C * a.J * 4);
  a.S = (double *)p;
  p += al((size_t)a.J * a.J * 8);
  a.V = (double *)p;
  p += al((size_t)a.J * a.J * 8);
  a.rot = p;
  p += al((size_t)(a.J / 2) * sizeof(Rot));
  a.done = (int *)p;
  p += al(sizeof(int));
  if (!a.ids) a.ids = (uint8_t *)p;
}

cudaError_t calibrate_launch(const CalibArgs &a, cudaStream_t st) {
  return a.prec == PREC_F32 ? calibrate_t<float>(a, st) : calibrate_t<__nv_bfloat16>(a, st);
}

}  // namespace nanokv
