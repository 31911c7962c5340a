// Tensor-core encode (NanoKV Fig. 4(b)): for each token x,
//     G = x [C | E]^T           (a GEMM, N = C + r, fp32)
//     a = argmin_j |c_j|^2 - 2 G[j]          (= argmin |x - c_j|^2)
//     y = G[C + k] - (E c_a)[k]              (= E (x - c_a))
//     s = fp16(max|y| / 7),  code = clamp(rint(y / s), -7, 7)
// The tables E c_j and |c_j|^2 come from nanokv_codec_prepare.  Both
// branches (K and V) run in one launch (grid.y).
// G is accumulated per 64-wide K block into one of two TMEM buffers and the
// blocks are summed in fp32 registers by the epilogue, so no fp32
// accumulation chain is longer than one block on the tensor core; codes and
// ids are decided on values as accurate as a plain fp32 dot product.
#include "tc_common.cuh"

namespace nanokv {

using namespace sm100;
using namespace tc;

#ifdef NANOKV_TRACE
// clock64 events of both CTAs of the first cluster of the 2-CTA kernel
__device__ unsigned long long g_enc_trace[2][8][32];
#define ENC_TRACE(ev, j)                                                                             \
  do {                                                                                               \
    if (blockIdx.x < 2 && blockIdx.y == 0 && (j) < 32) g_enc_trace[blockIdx.x][ev][j] = clock64();  \
  } while (0)
#else
#define ENC_TRACE(ev, j) \
  do {                   \
  } while (0)
#endif

namespace {

constexpr uint32_t kA = 128 * 64 * 2;  // token tile [128 x 64] bf16

struct EncArgs {
  const float *aux[2];  // [C][r] E c_j, then [C] |c_j|^2
  uint8_t *ids[2];
  uint8_t *codes[2];
  __half *scales[2];
  int64_t T;
  int J, r, C;
  unsigned *err;
};

// Small codecs (C <= 64, r in {64, 128, 192}), the columns of G = x [C | E]^T
// split over a 2-CTA cluster per 128-token tile so that a chunk of 4680 tokens
// per branch fills all SMs and every CTA issues one MMA per K step:
//   CTA 0   centers (padded to 64 rows; rows >= C read as zero) and E rows [0, P0)
//   CTA 1   E rows [P0, r)
// with P0 chosen so both sides have about the same N.  Each side accumulates
// its columns per 64-wide K block into one of two TMEM buffers and sums the
// blocks in fp32 registers.  CTA 0 finds the nearest center and hands the id
// to CTA 1 through distributed shared memory; the two exchange their row
// maxima the same way, so both derive the same scale and each packs its own
// codes.  One MMA per K step reads the token tile once, and each CTA moves
// the token tile plus half the [C | E] tile per K block (32 KB).  The K loop
// runs at the rate TMA delivers those bytes to the SM; the tail after it
// (argmin, hand-off, E c_a, scale, packing) is kept short by staging this
// CTA's columns of the E c table in shared memory while the loop runs.
//   warp 0      TMA: token tile and this CTA's [C | E] rows per K block
//   warp 1      MMA issuer
//   warps 2,3   stage |c|^2 and this CTA's columns of E c into shared memory
//   warps 4..7  epilogue, thread = token (TMEM lane)
constexpr int SSTG = 5;

template <int R>
struct SplitCols {
  static constexpr int P0 = ((R - 64) / 2) / 32 * 32;  // E rows on CTA 0: 0, 32, 64 for r = 64, 128, 192
  static constexpr int N0 = 64 + P0;                   // CTA 0: padded centers + E rows [0, P0)
  static constexpr int N1 = R - P0;                    // CTA 1: E rows [P0, r)
  static constexpr int ECS = N1 + 4;                   // row stride of the staged E c slice (floats)
  static_assert(N0 % 32 == 0 && N1 % 32 == 0 && N0 <= 128 && N1 <= 128, "column split");
};

struct EncSBars {
  uint64_t full[SSTG], empty[SSTG], part_full[2], part_empty[2], ec_full, ids_full, max_full;
  uint32_t tmem_base;
  int abort;
  uint32_t ids[128];     // CTA 1: center id of each row, written by CTA 0
  float peer_max[128];   // the other CTA's row maxima
};

template <int R>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(256, 1)
    tc_encode_split_kernel(const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmC0,
                           const __grid_constant__ CUtensorMap tmEa0, const __grid_constant__ CUtensorMap tmEb0,
                           const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmC1,
                           const __grid_constant__ CUtensorMap tmEa1, const __grid_constant__ CUtensorMap tmEb1,
                           const EncArgs A) {
  using S = SplitCols<R>;
  extern __shared__ uint8_t smraw[];
  uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  constexpr uint32_t kBs = 128 * 128;  // up to 128 rows x 64 bf16
  uint8_t *sA = sm;
  uint8_t *sB = sA + SSTG * kA;
  float *sEC = (float *)(sB + SSTG * kBs);  // [C][ECS] this CTA's columns of E c_j
  float *sCN = sEC + A.C * S::ECS;          // [C] |c_j|^2 (CTA 0)
  __shared__ EncSBars B;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int br = blockIdx.y;
  const CUtensorMap *tmX = br ? &tmX1 : &tmX0;
  const int64_t t0 = (int64_t)(blockIdx.x >> 1) * 128;
  const int nkb = A.J / 64;
  const int C = A.C;
  const int ncols = rank ? S::N1 : S::N0;
  volatile int *abort = &B.abort;
  unsigned *err = A.err;
  constexpr uint32_t tmem_cols = 256;  // two per-block buffers of up to 128 columns
  if (threadIdx.x == 0) ENC_TRACE(5, 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < SSTG; ++i) { mbar_init(&B.full[i], 1); mbar_init(&B.empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&B.part_full[i], 1); mbar_init(&B.part_empty[i], 4); }
    mbar_init(&B.ec_full, 64);
    mbar_init(&B.ids_full, 128);
    mbar_init(&B.max_full, 128);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&B.tmem_base, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before any remote access: every
  // thread arrives here and waits before its first remote access (epilogue)
  // or at the end (the other warps)
  cluster_arrive();
  tc_fence_after();
  const uint32_t tbase = B.tmem_base;
  if (threadIdx.x == 0) ENC_TRACE(5, 1);

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap *tmB0 = rank ? (br ? &tmEb1 : &tmEb0) : (br ? &tmC1 : &tmC0);
      const CUtensorMap *tmB1 = br ? &tmEa1 : &tmEa0;  // CTA 0's E rows [0, P0)
      prefetch_tmap(tmX);
      prefetch_tmap(tmB0);
      if (rank == 0 && S::P0 > 0) prefetch_tmap(tmB1);
      const uint32_t bytes = kA + (uint32_t)ncols * 128;
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % SSTG;
        if (kb >= SSTG && !mbar_wait(&B.empty[s], ((kb / SSTG) - 1) & 1, abort, err)) break;
        ENC_TRACE(4, kb);
        mbar_arrive_expect_tx(&B.full[s], bytes);
        tma_load_2d(sA + s * kA, tmX, kb * 64, (int)t0, &B.full[s]);
        if (rank == 0) {
          tma_load_2d(sB + s * kBs, tmB0, kb * 64, 0, &B.full[s]);
          if (S::P0 > 0) tma_load_2d(sB + s * kBs + 64 * 128, tmB1, kb * 64, 0, &B.full[s]);
        } else {
          tma_load_2d(sB + s * kBs, tmB0, kb * 64, S::P0, &B.full[s]);
        }
        issued = kb + 1;
      }
      for (int kb = (issued > SSTG ? issued - SSTG : 0); kb < issued; ++kb)
        mbar_wait(&B.full[kb % SSTG], (kb / SSTG) & 1, nullptr, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, ncols, false, false);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % SSTG, pb = kb & 1;
        if (!mbar_wait(&B.full[s], (kb / SSTG) & 1, abort, err)) break;
        if (kb >= 2 && !mbar_wait(&B.part_empty[pb], ((kb >> 1) - 1) & 1, abort, err)) break;
        ENC_TRACE(0, kb);
        tc_fence_after();
        const uint32_t a = smem_u32(sA + s * kA), b = smem_u32(sB + s * kBs);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ss(tbase + pb * 128, sdesc_sw128(a + 32 * k, 16, 1024), sdesc_sw128(b + 32 * k, 16, 1024), idesc,
                 k > 0);
        mma_commit(&B.empty[s]);
        mma_commit(&B.part_full[pb]);
      }
    }
  } else if (warp < 4) {
    // E c slice for this CTA's projection columns, rows padded to ECS floats
    const int ecol = rank ? S::P0 : 0, ncol = rank ? S::N1 : S::P0;
    const int i0 = threadIdx.x - 64, n4 = ncol / 4;
    for (int i = i0; i < C * n4; i += 64) {
      const int j = i / n4, k4 = i - j * n4;
      const float4 v = __ldg(reinterpret_cast<const float4 *>(A.aux[br] + (size_t)j * R + ecol) + k4);
      *reinterpret_cast<float4 *>(sEC + j * S::ECS + 4 * k4) = v;
    }
    if (rank == 0)
      for (int i = i0; i < C; i += 64) sCN[i] = A.aux[br][(size_t)C * R + i];
    mbar_arrive(&B.ec_full);
  } else {
    const int row = (warp - 4) * 32 + lane;
    const int64_t t = t0 + row;
    constexpr int NM = S::N0 > S::N1 ? S::N0 : S::N1;
    float acc[NM];
#pragma unroll
    for (int k = 0; k < NM; ++k) acc[k] = 0.f;
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      const int pb = kb & 1;
      if (!mbar_wait(&B.part_full[pb], (kb >> 1) & 1, abort, err)) { ok = false; break; }
      if (row == 0) ENC_TRACE(1, kb);
      tc_fence_after();
      uint32_t g[32];
#pragma unroll
      for (int k0 = 0; k0 < NM; k0 += 32) {
        if (k0 < ncols) {
          tmem_ld32(tmem_lane_addr(tbase, warp, pb * 128 + k0), g);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[k0 + i] += __uint_as_float(g[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.part_empty[pb]);
      if (row == 0) ENC_TRACE(2, kb);
    }
    if (row == 0) ENC_TRACE(3, 0);
    cluster_wait();
    if (ok) ok = mbar_wait(&B.ec_full, 0, abort, err);
    // nearest center on CTA 0 (strict < keeps the lowest index), handed to CTA 1
    int a = 0;
    if (rank == 0) {
      if (ok) {
        float best = INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j < C) {
            const float sc = fmaf(-2.f, acc[j], sCN[j]);
            if (sc < best) { best = sc; a = j; }
          }
        }
      }
      st_cluster_u32(mapa(smem_u32(&B.ids[row]), peer), (uint32_t)a);
      mbar_arrive_cluster(mapa(smem_u32(&B.ids_full), peer));
    } else {
      if (ok) ok = mbar_wait_cluster(&B.ids_full, 0, abort, err);
      if (ok) a = (int)B.ids[row];
    }
    if (row == 0) ENC_TRACE(3, 1);
    // y = E x - E c_a over this CTA's projection columns
    constexpr int Y0 = 64;  // first projection column on CTA 0
    const int ecol0 = rank ? S::P0 : 0;  // in E rows
    float m = 0.f;
    if (ok) {
      const float4 *e4 = reinterpret_cast<const float4 *>(sEC + a * S::ECS);
      if (rank == 0) {
#pragma unroll
        for (int k4 = 0; k4 < S::P0 / 4; ++k4) {
          const float4 e = e4[k4];
          acc[Y0 + 4 * k4 + 0] -= e.x;
          acc[Y0 + 4 * k4 + 1] -= e.y;
          acc[Y0 + 4 * k4 + 2] -= e.z;
          acc[Y0 + 4 * k4 + 3] -= e.w;
        }
#pragma unroll
        for (int k = 0; k < S::P0; ++k) m = fmaxf(m, fabsf(acc[Y0 + k]));
      } else {
#pragma unroll
        for (int k4 = 0; k4 < S::N1 / 4; ++k4) {
          const float4 e = e4[k4];
          acc[4 * k4 + 0] -= e.x;
          acc[4 * k4 + 1] -= e.y;
          acc[4 * k4 + 2] -= e.z;
          acc[4 * k4 + 3] -= e.w;
        }
#pragma unroll
        for (int k = 0; k < S::N1; ++k) m = fmaxf(m, fabsf(acc[k]));
      }
    }
    // row maximum over both CTAs
    st_cluster_u32(mapa(smem_u32(&B.peer_max[row]), peer), __float_as_uint(m));
    mbar_arrive_cluster(mapa(smem_u32(&B.max_full), peer));
    if (ok) ok = mbar_wait_cluster(&B.max_full, 0, abort, err);
    if (row == 0) ENC_TRACE(3, 2);
    if (ok) {
      m = fmaxf(m, B.peer_max[row]);
      const __half sh = __float2half_rn(m / 7.0f);
      const float sf = __half2float(sh);
      // y * (1/s) with a correctly rounded reciprocal, as in the other encode kernels
      const float inv = sf > 0.f ? __frcp_rn(sf) : 0.f;
      uint8_t *crow = A.codes[br] + t * (R / 2) + ecol0 / 2;
      auto pack8 = [&](int k) {
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int code = (int)fminf(7.f, fmaxf(-7.f, rintf(acc[k + i] * inv)));
          w |= (uint32_t)(code & 0xF) << (4 * i);
        }
        return w;
      };
      if (t < A.T) {
        // register indices stay compile-time: one loop per side
        if (rank == 0) {
#pragma unroll
          for (int k0 = 0; k0 < S::P0; k0 += 32)
            *reinterpret_cast<uint4 *>(crow + k0 / 2) =
                make_uint4(pack8(Y0 + k0), pack8(Y0 + k0 + 8), pack8(Y0 + k0 + 16), pack8(Y0 + k0 + 24));
        } else {
#pragma unroll
          for (int k0 = 0; k0 < S::N1; k0 += 32)
            *reinterpret_cast<uint4 *>(crow + k0 / 2) =
                make_uint4(pack8(k0), pack8(k0 + 8), pack8(k0 + 16), pack8(k0 + 24));
        }
        if (rank == 0) {
          A.ids[br][t] = (uint8_t)a;
          A.scales[br][t] = sh;
        }
      }
    }
    if (row == 0) ENC_TRACE(3, 3);
  }
  if (warp < 4) cluster_wait();
  tc_fence_before();
  __syncthreads();
  // the peer's stores and arrives into this CTA's shared memory are done
  // before either CTA exits
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, tmem_cols);
  }
}

// Large codecs (C up to 256, r up to 384): G = x [C | E]^T no longer fits in
// 512 TMEM columns next to the per-block projection buffers, and E x no longer
// fits in one thread's registers.  The K loop therefore runs once per pass:
//   pass 0        x C^T, N = C, accumulated in TMEM columns [0, C)
//   pass 1 + p    x E_p^T for the p-th 128-row slice of E, per 64-wide K block
//                 into one of two TMEM buffers (columns [256, 384), [384, 512)),
//                 summed in fp32 registers as in the small-codec kernel
// The token tile is re-read once per pass (from L2: a 128-token tile of a
// 3072-wide x is 768 KB).  The epilogue is two warpgroups, each owning half of
// every slice's columns; a finished slice (y - E c_a) is parked in TMEM
// columns [128 p, 128 p + 128), where pass 0's center scores were, until the
// row maximum, and so the scale, is known.
//   warp 0       TMA: token tile and [centers] or [E slice] tile per K block
//   warp 1       MMA issuer
//   warps 4..11  epilogue: thread (row, half) with row = lane quarter of TMEM
constexpr int LSTG = 4;
constexpr int kRS = 128;  // E rows (projection columns) per pass

struct EncLBars {
  uint64_t full[LSTG], empty[LSTG], acc_full, part_full[2], part_empty[2], cen_read, max_full;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(384, 1)
    tc_encode_large_kernel(const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmC0,
                           const __grid_constant__ CUtensorMap tmE0, const __grid_constant__ CUtensorMap tmX1,
                           const __grid_constant__ CUtensorMap tmC1, const __grid_constant__ CUtensorMap tmE1,
                           const EncArgs A) {
  extern __shared__ uint8_t smraw[];
  uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  const int C = A.C, R = A.r;
  const uint32_t kBmax = (uint32_t)(C > kRS ? C : kRS) * 128;
  uint8_t *sA = sm;
  uint8_t *sB = sA + LSTG * kA;
  float *sCN = (float *)(sB + LSTG * kBmax);  // [C] |c_j|^2
  float *sMax = sCN + C;                      // [2][128] per-half row maxima
  __shared__ EncLBars B;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int br = blockIdx.y;
  const CUtensorMap *tmX = br ? &tmX1 : &tmX0;
  const CUtensorMap *tmC = br ? &tmC1 : &tmC0;
  const CUtensorMap *tmE = br ? &tmE1 : &tmE0;
  const int64_t t0 = (int64_t)blockIdx.x * 128;
  const int nkb = A.J / 64;
  const int ns = (R + kRS - 1) / kRS;  // projection passes
  volatile int *abort = &B.abort;
  unsigned *err = A.err;
  constexpr uint32_t tmem_cols = 512;
  constexpr uint32_t kPartCol = 256;

  if (threadIdx.x == 0) {
    for (int i = 0; i < LSTG; ++i) { mbar_init(&B.full[i], 1); mbar_init(&B.empty[i], 1); }
    mbar_init(&B.acc_full, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&B.part_full[i], 1); mbar_init(&B.part_empty[i], 8); }
    mbar_init(&B.cen_read, 8);
    mbar_init(&B.max_full, 8);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&B.tmem_base, tmem_cols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < C; i += blockDim.x) sCN[i] = A.aux[br][(size_t)C * R + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = B.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(tmX);
      prefetch_tmap(tmC);
      prefetch_tmap(tmE);
      int q = 0;
      bool ok = true;
      for (int p = 0; p <= ns && ok; ++p) {
        const uint32_t bbytes = p == 0 ? (uint32_t)C * 128 : (uint32_t)kRS * 128;
        for (int kb = 0; kb < nkb; ++kb, ++q) {
          const int s = q % LSTG;
          if (q >= LSTG && !mbar_wait(&B.empty[s], ((q / LSTG) - 1) & 1, abort, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&B.full[s], kA + bbytes);
          tma_load_2d(sA + s * kA, tmX, kb * 64, (int)t0, &B.full[s]);
          if (p == 0)
            tma_load_2d(sB + s * kBmax, tmC, kb * 64, 0, &B.full[s]);
          else
            tma_load_2d(sB + s * kBmax, tmE, kb * 64, (p - 1) * kRS, &B.full[s]);
        }
      }
      // every issued copy lands before the CTA can exit
      for (int i = (q > LSTG ? q - LSTG : 0); i < q; ++i) mbar_wait(&B.full[i % LSTG], (i / LSTG) & 1, nullptr, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      int q = 0;
      const uint32_t idc = idesc_bf16(128, C, false, false);
      for (int kb = 0; kb < nkb; ++kb, ++q) {
        const int s = q % LSTG;
        if (!mbar_wait(&B.full[s], (q / LSTG) & 1, abort, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a = smem_u32(sA + s * kA), b = smem_u32(sB + s * kBmax);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ss(tbase, sdesc_sw128(a + 32 * k, 16, 1024), sdesc_sw128(b + 32 * k, 16, 1024), idc,
                 (kb > 0 || k > 0));
        mma_commit(&B.empty[s]);
      }
      if (ok) mma_commit(&B.acc_full);
      int g = 0;  // projection block counter across passes
      for (int p = 0; p < ns && ok; ++p) {
        const int width = R - p * kRS < kRS ? R - p * kRS : kRS;
        const uint32_t ide = idesc_bf16(128, width, false, false);
        for (int kb = 0; kb < nkb; ++kb, ++q, ++g) {
          const int s = q % LSTG, pb = g & 1;
          if (!mbar_wait(&B.full[s], (q / LSTG) & 1, abort, err)) { ok = false; break; }
          if (g >= 2 && !mbar_wait(&B.part_empty[pb], ((g >> 1) - 1) & 1, abort, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(sA + s * kA), b = smem_u32(sB + s * kBmax);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss(tbase + kPartCol + pb * kRS, sdesc_sw128(a + 32 * k, 16, 1024),
                   sdesc_sw128(b + 32 * k, 16, 1024), ide, k > 0);
          mma_commit(&B.empty[s]);
          mma_commit(&B.part_full[pb]);
        }
      }
    }
  } else if (warp >= 4) {
    const int row = (warp & 3) * 32 + lane;
    const int half = (warp - 4) >> 2;  // columns [64 half, 64 half + 64) of every slice
    const int64_t t = t0 + row;
    bool ok = mbar_wait(&B.acc_full, 0, abort, err);
    int a = 0;
    float m = 0.f;
    if (ok) {
      tc_fence_after();
      uint32_t g[32];
      // nearest center: argmin |c_j|^2 - 2 x.c_j, strict < keeps the lowest index
      float best = INFINITY;
      for (int c0 = 0; c0 < C; c0 += 32) {
        tmem_ld32(tmem_lane_addr(tbase, warp, c0), g);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (c0 + i < C) {
            const float sc = fmaf(-2.f, __uint_as_float(g[i]), sCN[c0 + i]);
            if (sc < best) { best = sc; a = c0 + i; }
          }
        }
      }
    }
    // both halves read the center scores of a row before either parks a
    // slice over them
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&B.cen_read);
    bool cen_free = false;
    const float *ec = A.aux[br] + (size_t)a * R;
    float y[64];
    int g = 0;
    int last_w = 0;  // this thread's column count in the last slice
    for (int p = 0; p < ns && ok; ++p) {
      const int width = R - p * kRS < kRS ? R - p * kRS : kRS;
      const int col0 = half * 64;
      const bool mine = col0 < width;  // a 64-wide last slice belongs to half 0
#pragma unroll
      for (int k = 0; k < 64; ++k) y[k] = 0.f;
      for (int kb = 0; kb < nkb; ++kb, ++g) {
        const int pb = g & 1;
        if (!mbar_wait(&B.part_full[pb], (g >> 1) & 1, abort, err)) { ok = false; break; }
        tc_fence_after();
        if (mine) {
          uint32_t v[32];
#pragma unroll
          for (int k0 = 0; k0 < 64; k0 += 32) {
            tmem_ld32(tmem_lane_addr(tbase, warp, kPartCol + pb * kRS + col0 + k0), v);
#pragma unroll
            for (int i = 0; i < 32; ++i) y[k0 + i] += __uint_as_float(v[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.part_empty[pb]);
      }
      if (!ok || !mine) continue;
      // y = E x - E c_a for this slice
      const float4 *e4 = reinterpret_cast<const float4 *>(ec + p * kRS + col0);
#pragma unroll
      for (int k4 = 0; k4 < 16; ++k4) {
        const float4 e = __ldg(e4 + k4);
        y[4 * k4 + 0] -= e.x;
        y[4 * k4 + 1] -= e.y;
        y[4 * k4 + 2] -= e.z;
        y[4 * k4 + 3] -= e.w;
      }
#pragma unroll
      for (int k = 0; k < 64; ++k) m = fmaxf(m, fabsf(y[k]));
      if (p + 1 < ns) {
        // park the slice where pass 0's center scores were
        if (!cen_free) {
          if (!(cen_free = mbar_wait(&B.cen_read, 0, abort, err))) { ok = false; continue; }
          tc_fence_after();
        }
#pragma unroll
        for (int k0 = 0; k0 < 64; k0 += 16) {
          uint32_t v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(y[k0 + i]);
          tmem_st16(tmem_lane_addr(tbase, warp, p * kRS + col0 + k0), v);
        }
        tmem_st_wait();
      } else {
        last_w = 64;
      }
    }
    // row maximum over both halves
    sMax[half * 128 + row] = m;
    __syncwarp();
    if (lane == 0) mbar_arrive(&B.max_full);
    if (ok) ok = mbar_wait(&B.max_full, 0, abort, err);
    if (ok) {
      m = fmaxf(sMax[row], sMax[128 + row]);
      const __half sh = __float2half_rn(m / 7.0f);
      const float sf = __half2float(sh);
      // y * (1/s) with a correctly rounded reciprocal, as in the small-codec kernel
      const float inv = sf > 0.f ? __frcp_rn(sf) : 0.f;
      uint8_t *crow = A.codes[br] + t * (R / 2);
      auto pack8 = [&](const float *v) {
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int code = (int)fminf(7.f, fmaxf(-7.f, rintf(v[i] * inv)));
          acc |= (uint32_t)(code & 0xF) << (4 * i);
        }
        return acc;
      };
      for (int p = 0; p + 1 < ns; ++p) {
#pragma unroll
        for (int k0 = 0; k0 < 64; k0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem_lane_addr(tbase, warp, p * kRS + half * 64 + k0), v);
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          const uint4 w = make_uint4(pack8(f), pack8(f + 8), pack8(f + 16), pack8(f + 24));
          if (t < A.T) *reinterpret_cast<uint4 *>(crow + (p * kRS + half * 64 + k0) / 2) = w;
        }
      }
      if (last_w) {
        const int p = ns - 1;
#pragma unroll
        for (int k0 = 0; k0 < 64; k0 += 32) {
          const uint4 w = make_uint4(pack8(y + k0), pack8(y + k0 + 8), pack8(y + k0 + 16), pack8(y + k0 + 24));
          if (t < A.T) *reinterpret_cast<uint4 *>(crow + (p * kRS + half * 64 + k0) / 2) = w;
        }
      }
      if (half == 0 && t < A.T) {
        A.ids[br][t] = (uint8_t)a;
        A.scales[br][t] = sh;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, tmem_cols);
  }
}

// EC[j][k] = E[k] . c_j and |c_j|^2 in fp32: a small GEMM of the codec's
// centers against its encoder (2 C r J flops; reads dominate), once per codec.

// 8 consecutive parameters as they are stored: 16 bytes of bf16 or 32 of fp32
template <typename TP>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) { w = __ldg(reinterpret_cast<const uint4 *>(p)); }
  __device__ __forceinline__ void zero() { w = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ float get(int q) const {
    const uint32_t u = q < 2 ? w.x : q < 4 ? w.y : q < 6 ? w.z : w.w;
    return __uint_as_float((q & 1) ? (u & 0xffff0000u) : (u << 16));
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float *p) {
    a = __ldg(reinterpret_cast<const float4 *>(p));
    b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ float get(int q) const {
    const float4 &v = q < 4 ? a : b;
    const int k = q & 3;
    return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
  }
};

// E c_j and |c_j|^2, one 8 x 8 tile of (center, encoder row) pairs per block.
// Each thread loads its 8-element slices of the tile's 8 center rows and 8
// encoder rows (every load of a pass in flight at once: one pass covers
// J = 1536), kept as stored, and forms the 64 partial dot products in fp32
// element by element; the block then sums them in a fixed order: a shuffle
// reduce-scatter inside each warp (after which lane L holds the warp's sums
// of products 2L and 2L + 1), then the warps in order.  The norms come from
// the blocks of the first column.  Two blocks fit an SM.
constexpr int kPrepT = 8;    // centers (and encoder rows) per tile
constexpr int kPrepNT = 192;  // threads per block

template <typename TP>
__global__ void __launch_bounds__(kPrepNT, sizeof(TP) == 2 ? 2 : 1)
    codec_prepare_kernel(const TP *__restrict__ cen, const TP *__restrict__ E, int C, int r, int J,
                         float *__restrict__ aux) {
  constexpr int NW = kPrepNT / 32;
  __shared__ float red[NW][kPrepT * kPrepT + kPrepT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k0 = blockIdx.x * kPrepT, j0 = blockIdx.y * kPrepT;
  const bool norms = blockIdx.x == 0;
  float acc[kPrepT * kPrepT], nrm[kPrepT];
#pragma unroll
  for (int i = 0; i < kPrepT * kPrepT; ++i) acc[i] = 0.f;
#pragma unroll
  for (int a = 0; a < kPrepT; ++a) nrm[a] = 0.f;
  for (int i = threadIdx.x * 8; i < J; i += kPrepNT * 8) {
    Raw8<TP> c[kPrepT], e[kPrepT];
#pragma unroll
    for (int a = 0; a < kPrepT; ++a) {
      if (j0 + a < C) c[a].load(cen + (size_t)(j0 + a) * J + i);
      else c[a].zero();
    }
#pragma unroll
    for (int b = 0; b < kPrepT; ++b) {
      if (k0 + b < r) e[b].load(E + (size_t)(k0 + b) * J + i);
      else e[b].zero();
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float cq[kPrepT], eq[kPrepT];
#pragma unroll
      for (int a = 0; a < kPrepT; ++a) cq[a] = c[a].get(q);
#pragma unroll
      for (int b = 0; b < kPrepT; ++b) eq[b] = e[b].get(q);
#pragma unroll
      for (int a = 0; a < kPrepT; ++a) {
        nrm[a] = fmaf(cq[a], cq[a], nrm[a]);
#pragma unroll
        for (int b = 0; b < kPrepT; ++b) acc[a * kPrepT + b] = fmaf(cq[a], eq[b], acc[a * kPrepT + b]);
      }
    }
  }
  // reduce-scatter over the warp: at offset o each lane keeps the half of its
  // values selected by its lane bit o and adds the partner's copy of that half
#pragma unroll
  for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = hi ? acc[i] : acc[i + n];
      const float keep = hi ? acc[i + n] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  red[warp][2 * lane] = acc[0];
  red[warp][2 * lane + 1] = acc[1];
  if (norms) {
#pragma unroll
    for (int a = 0; a < kPrepT; ++a) {
      const float v = warp_sum(nrm[a]);
      if (lane == 0) red[warp][kPrepT * kPrepT + a] = v;
    }
  }
  __syncthreads();
  const int t = threadIdx.x;
  if (t < kPrepT * kPrepT + (norms ? kPrepT : 0)) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += red[w][t];
    if (t < kPrepT * kPrepT) {
      const int a = t / kPrepT, b = t % kPrepT;
      if (j0 + a < C && k0 + b < r) aux[(size_t)(j0 + a) * r + k0 + b] = v;
    } else if (j0 + t - kPrepT * kPrepT < C) {
      aux[(size_t)C * r + j0 + t - kPrepT * kPrepT] = v;
    }
  }
}

}  // namespace

size_t codec_aux_bytes(const Codec &c) {
  return (((size_t)c.C * c.r + c.C) * sizeof(float) + 255) & ~(size_t)255;
}

cudaError_t codec_prepare(const Codec &c, void *aux, cudaStream_t st) {
  const dim3 grid((unsigned)((c.r + kPrepT - 1) / kPrepT), (unsigned)((c.C + kPrepT - 1) / kPrepT));
  if (c.prec == PREC_F32)
    codec_prepare_kernel<float><<<grid, kPrepNT, 0, st>>>((const float *)c.centers, (const float *)c.E, c.C, c.r,
                                                          c.H * c.d, (float *)aux);
  else
    codec_prepare_kernel<__nv_bfloat16><<<grid, kPrepNT, 0, st>>>(
        (const __nv_bfloat16 *)c.centers, (const __nv_bfloat16 *)c.E, c.C, c.r, c.H * c.d, (float *)aux);
  return cudaGetLastError();
}

// the 2-CTA kernel's column split needs C <= 64 (one padded 64-row center
// box) and r in {64, 128, 192}
static bool enc_small(const Codec &c) { return (c.r == 64 || c.r == 128 || c.r == 192) && c.C <= 64; }

bool tc_encode_supported(const Codec &c) {
  if (!(c.prec == PREC_BF16 && c.aux && (c.H * c.d) % 64 == 0 && c.C % 16 == 0 && c.C >= 16)) return false;
  return enc_small(c) || (c.r % 64 == 0 && c.r >= 64 && c.r <= 384 && c.C <= 256);
}

static size_t enc_large_smem(const Codec &c) {
  const size_t kb = (size_t)(c.C > kRS ? c.C : kRS) * 128;
  return LSTG * (kA + kb) + ((size_t)c.C + 256) * sizeof(float) + 1024;
}

static size_t enc_split_smem(const Codec &c) {
  const int P0 = ((c.r - 64) / 2) / 32 * 32, ecs = c.r - P0 + 4;
  return SSTG * (kA + 128 * 128) + (size_t)c.C * (ecs + 1) * sizeof(float) + 1024;
}

template <int R>
static cudaError_t launch_split(CUtensorMap (&m)[2][4], const EncArgs &a, int64_t T, int nbranch, size_t smem,
                                cudaStream_t st) {
  static_assert(SplitCols<R>::ECS == R - SplitCols<R>::P0 + 4, "staged E c stride");
  ensure_smem((const void *)tc_encode_split_kernel<R>, (int)smem);
  dim3 grid((unsigned)(2 * ((T + 127) / 128)), (unsigned)nbranch);
  tc_encode_split_kernel<R><<<grid, 256, smem, st>>>(m[0][0], m[0][1], m[0][2], m[0][3], m[1][0], m[1][1],
                                                      m[1][2], m[1][3], a);
  return cudaGetLastError();
}

static void fill_args(EncArgs &a, const Codec *c, uint8_t *const *ids, uint8_t *const *codes,
                      void *const *scales, int nbranch, int64_t T) {
  for (int b = 0; b < nbranch; ++b) {
    a.aux[b] = (const float *)c[b].aux;
    a.ids[b] = ids[b];
    a.codes[b] = codes[b];
    a.scales[b] = (__half *)scales[b];
  }
  a.T = T;
  a.J = c[0].H * c[0].d;
  a.r = c[0].r;
  a.C = c[0].C;
  a.err = error_word_ptr();
}

static cudaError_t tc_encode_split(const Codec *c, const void *const *x, int64_t T, uint8_t *const *ids,
                                   uint8_t *const *codes, void *const *scales, int nbranch, cudaStream_t st) {
  CUtensorMap m[2][4];
  const int J = c[0].H * c[0].d, r = c[0].r;
  const int P0 = ((r - 64) / 2) / 32 * 32, N1 = r - P0;
  for (int b = 0; b < nbranch; ++b) {
    // x tile; centers (64-row box, rows >= C read as zero); E rows [0, P0) for
    // CTA 0 (the centers map stands in when P0 = 0); E rows [P0, r) for CTA 1
    if (!make_tmap_bf16_2d(&m[b][0], x[b], T, J, J, 128) ||
        !make_tmap_bf16_2d(&m[b][1], c[b].centers, c[b].C, J, J, 64) ||
        !(P0 == 0 ? (m[b][2] = m[b][1], true) : make_tmap_bf16_2d(&m[b][2], c[b].E, r, J, J, P0)) ||
        !make_tmap_bf16_2d(&m[b][3], c[b].E, r, J, J, N1))
      return cudaErrorInvalidValue;
  }
  if (nbranch == 1)
    for (int i = 0; i < 4; ++i) m[1][i] = m[0][i];
  EncArgs a{};
  fill_args(a, c, ids, codes, scales, nbranch, T);
  const size_t smem = enc_split_smem(c[0]);
  switch (r) {
    case 64: return launch_split<64>(m, a, T, nbranch, smem, st);
    case 128: return launch_split<128>(m, a, T, nbranch, smem, st);
    case 192: return launch_split<192>(m, a, T, nbranch, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t tc_encode_pair(const Codec *c, const void *const *x, int64_t T, uint8_t *const *ids,
                           uint8_t *const *codes, void *const *scales, int nbranch, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (enc_small(c[0])) return tc_encode_split(c, x, T, ids, codes, scales, nbranch, st);
  CUtensorMap m[2][3];
  const int J = c[0].H * c[0].d;
  for (int b = 0; b < nbranch; ++b) {
    if (!make_tmap_bf16_2d(&m[b][0], x[b], T, J, J, 128) ||
        !make_tmap_bf16_2d(&m[b][1], c[b].centers, c[b].C, J, J, c[b].C) ||
        !make_tmap_bf16_2d(&m[b][2], c[b].E, c[b].r, J, J, kRS))
      return cudaErrorInvalidValue;
  }
  if (nbranch == 1)
    for (int i = 0; i < 3; ++i) m[1][i] = m[0][i];
  EncArgs a{};
  fill_args(a, c, ids, codes, scales, nbranch, T);
  const size_t smem = enc_large_smem(c[0]);
  dim3 grid((unsigned)((T + 127) / 128), (unsigned)nbranch);
  ensure_smem((const void *)tc_encode_large_kernel, (int)smem);
  tc_encode_large_kernel<<<grid, 384, smem, st>>>(m[0][0], m[0][1], m[0][2], m[1][0], m[1][1], m[1][2], a);
  return cudaGetLastError();
}

#ifdef NANOKV_TRACE
extern "C" int nanokv_debug_enc_trace(void *host, size_t bytes) {
  if (bytes < sizeof(g_enc_trace)) return -1;
  return cudaMemcpyFromSymbol(host, g_enc_trace, sizeof(g_enc_trace)) == cudaSuccess ? 0 : -3;
}
#endif

}  // namespace nanokv
