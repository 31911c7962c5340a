// Tensor-core mixed-dimensional attention (NanoKV-Fast; abstract: reuse the
// stored coefficients; Fig. 4(d): reduce the queries, restore the output
// dimension) for codecs too large for the single-CTA kernel (r up to 384,
// up to 256 centers).  Per head h, with D_h the head's rows of D and c_{j,h}
// the head's slice of center j:
//   prologue  Q~ = Q D_{K,h}                                   (r per row)
//   per tile  S' = Q~ codes_K^T,  S2 = Q c_K[a]^T               (MMA)
//             z  = tau (s_K S' + S2)                (softmax, log2 units)
//             O~ += (P s_V) codes_V,  O_c += P c_V[a]           (MMA)
//   epilogue  O  = (O~ D_{V,h}^T + O_c) / l                    (MMA + add)
// The center terms are products with the gathered center rows of the tile's
// keys, exact in fp32 like the rest of the contraction.
//
// A cluster of two CTAs serves 128 query rows of one head with pair MMAs
// (tcgen05 cta_group::2, M = 128, issued by CTA 0): each CTA holds 64 query
// rows, and its accumulators take 64 rows over all 128 TMEM lanes in N / 2
// columns (lanes [0, 64): columns [0, N/2) of D; lanes [64, 128): [N/2, N)),
// which is what lets S', S2 (both double-buffered), O~ (r = 384) and O_c fit
// the 512 columns.  Every B operand is split by N between the CTAs: CTA c
// holds the key codes and key centers of keys [64c, 64c + 64) of each tile,
// the value codes of columns [128m + 64c, 128m + 64c + 64) of each 128-column
// block m, and the value centers of d rows [64c, 64c + 64).
// Roles (12 warps per CTA):
//   warp 0       TMEM allocation; TMA of Q, D_{K,h} (prologue), D_{V,h} (restore)
//   warp 1       CTA 0: MMA issue
//   warps 2, 3   key codes and key centers of this CTA's 64 keys
//   warps 4..7   value codes and value centers of all 128 keys
//   warps 8..11  softmax: thread l = TMEM lane: query row l & 63, key half l >> 6
// Codes are unpacked in the order (0,4,1,5,2,6,3,7) within each group of 8;
// Q~ is stored in that order and O~ is un-permuted before the restore.
// Every wait is bounded.
#include "tc_common.cuh"

namespace nanokv {

using namespace sm100;
using namespace tc;

namespace {

constexpr int DH = 128;
constexpr uint32_t kB64 = 64 * 64 * 2;    // [64 rows x 64] bf16 (8 KB)
constexpr uint32_t kB128 = 128 * 64 * 2;  // [128 rows x 64] bf16 (16 KB)
constexpr int kMaxR = 384;
constexpr uint32_t IDESC_KK = idesc_bf16(128, 128, false, false);  // pair, M = 128, A and B K-major
constexpr uint32_t IDESC_KM = idesc_bf16(128, 128, false, true);   // pair, M = 128, B MN-major
constexpr uint32_t TM_S1 = 0, TM_S2 = 128, TM_OT = 256, TM_COLS = 512;  // O_c at TM_OT + r / 2
constexpr uint16_t kBoth = 0x3;

struct PairArgs {
  const __nv_bfloat16 *Ck, *Cv;  // centers [C, J]
  const uint8_t *idk, *idv;      // [T]
  const uint8_t *codk, *codv;    // [T, r/2]
  const __half *sk, *sv;         // [T]
  int64_t t0, T, Tq;
  int H, r, Ck_n, Cv_n;
  float zscale;
  float *O, *L;
  unsigned *err;
  const int32_t *head_map;  // heads of grid y (nullptr: y is the head)
};

// barriers and small arrays, at the end of the dynamic shared memory
struct PairBars {
  uint64_t pro_full, pro_ready, qt_ready;
  uint64_t kc_full, kc_empty, vc_full;
  uint64_t s_full[2], s_free[2], p_full, pv_done;
  uint64_t xbar[2], lbar;
  uint64_t fin_a, fin_b_local, fin_b, fin_done, s_last;
  uint32_t tmem_base;
  int abort;
  float xmax[2][2][64];  // [tile parity][key half][row]
  float lsum[2][64];     // [key half][row]
  __half meta[4][2][64];  // [softmax warp][K / V scale][key of the warp's half]
};

__device__ __forceinline__ void arrive_leader(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(mapa(smem_u32(bar), 0)) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    tc_low_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDk,
                       const __grid_constant__ CUtensorMap tmDv, const PairArgs A) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  // The operand tiles need 1024-byte alignment.  This kernel has no static
  // shared memory, so the dynamic region starts aligned and the whole budget
  // goes to the tiles; should that ever not hold, fail cleanly (both CTAs
  // take the same branch before any barrier or TMEM use).
  if ((smem_u32(smraw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(A.err, ERRW_BOUNDS);
    return;
  }
  uint8_t *sm = smraw;
  const int r = A.r, nkb = r / 64, nm = r / 128;
  uint8_t *sQt = sm;                    // Q~ * zscale [64 rows x r] K-major; later O~ / l
  uint8_t *sQ = sQt + nkb * kB64;       // Q [64 rows x 128] K-major
  uint8_t *sKc = sQ + 2 * kB64;         // key codes [64 keys x r] K-major; later D_{V,h} half
  uint8_t *sCgK = sKc + nkb * kB64;     // key centers [64 keys x 128 d] K-major
  uint8_t *sVc = sCgK + 2 * kB64;       // value codes [128 keys x 64] MN-major per block m; first D_{K,h} halves
  uint8_t *sCgV = sVc + nm * kB128;     // value centers [128 keys x 64 d] MN-major
  uint8_t *sP = sCgV + kB128;           // P [64 rows x 128 keys] K-major
  uint8_t *sPs = sP + 2 * kB64;         // P s_V
  PairBars &B = *reinterpret_cast<PairBars *>(sPs + 2 * kB64);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int h = A.head_map ? A.head_map[blockIdx.y] : (int)blockIdx.y;
  const int64_t q0 = (int64_t)(blockIdx.x >> 1) * 128 + 64 * rank;  // this CTA's first query row
  const int ntiles = (int)((A.T + BN - 1) / BN);
  const int J = A.H * DH;
  const uint32_t TM_OC = TM_OT + r / 2;
  volatile int *abort = &B.abort;
  unsigned *err = A.err;

  if (threadIdx.x == 0) {
    mbar_init(&B.pro_full, 1);
    mbar_init(&B.pro_ready, 2);
    mbar_init(&B.qt_ready, 8);
    mbar_init(&B.kc_full, 4);
    mbar_init(&B.kc_empty, 1);
    mbar_init(&B.vc_full, 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.s_free[i], 8);
      mbar_init(&B.xbar[i], 4);
    }
    mbar_init(&B.p_full, 8);
    mbar_init(&B.pv_done, 1);
    mbar_init(&B.lbar, 4);
    mbar_init(&B.fin_a, 8);
    mbar_init(&B.fin_b_local, 1);
    mbar_init(&B.fin_b, 2);
    mbar_init(&B.fin_done, 1);
    mbar_init(&B.s_last, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc2(&B.tmem_base, TM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and TMEM ready before any remote access or MMA
  tc_fence_after();
  const uint32_t tbase = B.tmem_base;

  if (warp == 0) {
    // ---------------- TMA: Q and D_{K,h} halves; later D_{V,h} half ----------------
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmDk);
      prefetch_tmap(&tmDv);
      mbar_arrive_expect_tx(&B.pro_full, 2 * kB64 + nm * kB128);
      for (int k = 0; k < 2; ++k) tma_load_2d(sQ + k * kB64, &tmQ, h * DH + 64 * k, (int)q0, &B.pro_full);
      for (int m = 0; m < nm; ++m)
        tma_load_2d(sVc + m * kB128, &tmDk, 128 * m + 64 * (int)rank, h * DH, &B.pro_full);
      bool ok = mbar_wait(&B.pro_full, 0, abort, err);
      if (ok) arrive_leader(&B.pro_ready);
      // D_{V,h} rows [64c, 64c + 64) into the key-code buffer once the last
      // scores (its last readers) are done
      if (ok) ok = mbar_wait(&B.s_last, 0, abort, err);
      if (ok) {
        mbar_arrive_expect_tx(&B.fin_b_local, nkb * kB64);
        for (int kb = 0; kb < nkb; ++kb)
          tma_load_2d(sKc + kb * kB64, &tmDv, 64 * kb, h * DH + 64 * (int)rank, &B.fin_b_local);
        if (mbar_wait(&B.fin_b_local, 0, abort, err)) arrive_leader(&B.fin_b);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (CTA 0, for both) ----------------
    if (lane == 0 && rank == 0) {
      const uint32_t aQt = smem_u32(sQt), aQ = smem_u32(sQ), aKc = smem_u32(sKc), aCgK = smem_u32(sCgK);
      const uint32_t aVc = smem_u32(sVc), aCgV = smem_u32(sCgV), aP = smem_u32(sP), aPs = smem_u32(sPs);
      bool ok = mbar_wait(&B.pro_ready, 0, abort, err);
      if (ok) {
        // Q~ = Q D_{K,h}: per 128-column block m, N split between the CTAs
        tc_fence_after();
        for (int m = 0; m < nm; ++m)
#pragma unroll
          for (int ks = 0; ks < DH / 16; ++ks)
            mma2_ss(tbase + TM_OT + 64 * m, sdesc_sw128(aQ + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024),
                    sdesc_sw128(aVc + m * kB128 + ks * 2048, kB128, 1024), IDESC_KM, ks > 0);
        mma2_commit_mc(&B.pv_done, kBoth);  // phase 0: the prologue's reads of the value-code buffer
        ok = mbar_wait(&B.qt_ready, 0, abort, err);
      }
      // scores of tile js (S buffer js & 1, free once both CTAs' softmax read
      // tile js - 2) and values of tile jv, polled without blocking
      int js = 0, jv = 0;
      uint64_t t_last = globaltimer();
      while (ok && jv < ntiles) {
        bool progress = false;
        if (jv < js && mbar_test(&B.p_full, jv & 1) && mbar_test(&B.vc_full, jv & 1)) {
          tc_fence_after();
          for (int m = 0; m < nm; ++m)
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks)
              mma2_ss(tbase + TM_OT + 64 * m, sdesc_sw128(aPs + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024),
                      sdesc_sw128(aVc + m * kB128 + ks * 2048, kB128, 1024), IDESC_KM, (jv > 0 || ks > 0));
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma2_ss(tbase + TM_OC, sdesc_sw128(aP + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024),
                    sdesc_sw128(aCgV + ks * 2048, kB128, 1024), IDESC_KM, (jv > 0 || ks > 0));
          mma2_commit_mc(&B.pv_done, kBoth);
          ++jv;
          progress = true;
        }
        if (js < ntiles && mbar_test(&B.kc_full, js & 1) &&
            (js < 2 || mbar_test(&B.s_free[js & 1], ((js - 2) >> 1) & 1))) {
          tc_fence_after();
          const uint32_t d1 = tbase + TM_S1 + 64 * (js & 1), d2 = tbase + TM_S2 + 64 * (js & 1);
          for (int ks = 0; ks < r / 16; ++ks)
            mma2_ss(d1, sdesc_sw128(aQt + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024),
                    sdesc_sw128(aKc + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024), IDESC_KK, ks > 0);
#pragma unroll
          for (int ks = 0; ks < DH / 16; ++ks)
            mma2_ss(d2, sdesc_sw128(aQ + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024),
                    sdesc_sw128(aCgK + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024), IDESC_KK, ks > 0);
          mma2_commit_mc(&B.s_full[js & 1], kBoth);
          mma2_commit_mc(&B.kc_empty, kBoth);
          if (js == ntiles - 1) mma2_commit_mc(&B.s_last, kBoth);
          ++js;
          progress = true;
        }
        if (progress) {
          t_last = globaltimer();
        } else {
          if (*abort) { ok = false; break; }
          if (globaltimer() - t_last > kWaitLimitNs) {
            *abort = 1;
            atomicOr(err, ERRW_TIMEOUT);
            ok = false;
            break;
          }
        }
      }
      // restore: O_r = (O~ / l) D_{V,h}^T into the first S buffer
      if (ok && mbar_wait(&B.fin_a, 0, abort, err) && mbar_wait(&B.fin_b, 0, abort, err)) {
        tc_fence_after();
        for (int ks = 0; ks < r / 16; ++ks)
          mma2_ss(tbase + TM_S1, sdesc_sw128(aQt + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024),
                  sdesc_sw128(aKc + (ks >> 2) * kB64 + (ks & 3) * 32, 16, 1024), IDESC_KK, ks > 0);
        mma2_commit_mc(&B.fin_done, kBoth);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------- key codes and key centers of this CTA's 64 keys ----------------
    const int kq = (warp - 2) * 32 + lane;  // key within this CTA's half
    const int cw = r / 32;                  // uint4 words of packed codes per key
    for (int j = 0; j < ntiles; ++j) {
      const int64_t kk = (int64_t)j * BN + 64 * rank + kq;
      const bool valid = kk < A.T;
      const int64_t tt = A.t0 + (valid ? kk : A.T - 1);
      int a = (int)A.idk[tt];
      a = a < A.Ck_n ? a : A.Ck_n - 1;
      uint4 cod[kMaxR / 32];
      const uint4 *pk = reinterpret_cast<const uint4 *>(A.codk + tt * (r / 2));
#pragma unroll
      for (int q = 0; q < kMaxR / 32; ++q) cod[q] = (q < cw && valid) ? __ldg(pk + q) : make_uint4(0, 0, 0, 0);
      const uint4 *pc = reinterpret_cast<const uint4 *>(A.Ck + (size_t)a * J + (size_t)h * DH);
      uint4 cen[16];
#pragma unroll
      for (int g = 0; g < 16; ++g) cen[g] = __ldg(pc + g);
      if (j >= 1 && !mbar_wait(&B.kc_empty, (j - 1) & 1, abort, err)) break;
#pragma unroll
      for (int q = 0; q < kMaxR / 32; ++q) {
        if (q >= cw) break;
        const uint32_t w[4] = {cod[q].x, cod[q].y, cod[q].z, cod[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          st_shared_v4(smem_u32(sKc) + sw128_offset(kq, 32 * q + 8 * i, 64), unpack8(w[i]));
      }
#pragma unroll
      for (int g = 0; g < 16; ++g) st_shared_v4(smem_u32(sCgK) + sw128_offset(kq, 8 * g, 64), cen[g]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) arrive_leader(&B.kc_full);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- value codes (this CTA's columns) and value centers (its d half) ----------------
    const int t = (warp - 4) * 32 + lane;  // key of the tile
    for (int j = 0; j < ntiles; ++j) {
      const int64_t kk = (int64_t)j * BN + t;
      const bool valid = kk < A.T;
      const int64_t tt = A.t0 + (valid ? kk : A.T - 1);
      int a = (int)A.idv[tt];
      a = a < A.Cv_n ? a : A.Cv_n - 1;
      uint4 cod[2 * (kMaxR / 128)];
      const uint4 *pv = reinterpret_cast<const uint4 *>(A.codv + tt * (r / 2));
#pragma unroll
      for (int m = 0; m < kMaxR / 128; ++m) {
        // columns [128m + 64c, 128m + 64c + 64): 32 bytes at byte 64m + 32c
        const bool on = m < nm && valid;
        cod[2 * m] = on ? __ldg(pv + 4 * m + 2 * rank) : make_uint4(0, 0, 0, 0);
        cod[2 * m + 1] = on ? __ldg(pv + 4 * m + 2 * rank + 1) : make_uint4(0, 0, 0, 0);
      }
      const uint4 *pc = reinterpret_cast<const uint4 *>(A.Cv + (size_t)a * J + (size_t)h * DH + 64 * rank);
      uint4 cen[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) cen[g] = valid ? __ldg(pc + g) : make_uint4(0, 0, 0, 0);
      // the previous tile's value MMAs (or the prologue, which read D_{K,h}
      // from this buffer) are done
      if (!mbar_wait(&B.pv_done, j & 1, abort, err)) break;
#pragma unroll
      for (int m = 0; m < kMaxR / 128; ++m) {
        if (m >= nm) break;
        const uint32_t w[8] = {cod[2 * m].x,     cod[2 * m].y,     cod[2 * m].z,     cod[2 * m].w,
                               cod[2 * m + 1].x, cod[2 * m + 1].y, cod[2 * m + 1].z, cod[2 * m + 1].w};
#pragma unroll
        for (int g = 0; g < 8; ++g)
          st_shared_v4(smem_u32(sVc) + m * kB128 + sw128_offset(t, 8 * g, 128), unpack8(w[g]));
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) st_shared_v4(smem_u32(sCgV) + sw128_offset(t, 8 * g, 128), cen[g]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) arrive_leader(&B.vc_full);
    }
  } else {
    // ---------------- softmax: thread l -> query row l & 63, key half l >> 6 ----------------
    const int l = (warp - 8) * 32 + lane;
    const int row = l & 63, hk = l >> 6;
    const float zs = A.zscale;
    __half *meta = &B.meta[warp - 8][0][0];
    // Q~ * zscale -> bf16 in the unpack order, for this thread's row and
    // r columns [128m + 64 hk, +64) of each block m, once the prologue MMAs
    // (pv_done's first completion, multicast to both CTAs) are done
    bool ok = mbar_wait(&B.pv_done, 0, abort, err);
    if (ok) {
      tc_fence_after();
      for (int m = 0; m < nm; ++m) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_lane_addr(tbase, warp, TM_OT + 64 * m + 32 * c), v);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const float *f = reinterpret_cast<const float *>(v + 8 * g);
            const uint4 o = make_uint4(pack_bf16x2(f[0] * zs, f[4] * zs), pack_bf16x2(f[1] * zs, f[5] * zs),
                                       pack_bf16x2(f[2] * zs, f[6] * zs), pack_bf16x2(f[3] * zs, f[7] * zs));
            st_shared_v4(smem_u32(sQt) + sw128_offset(row, 128 * m + 64 * hk + 32 * c + 8 * g, 64), o);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&B.qt_ready);
    }
    RowState st{-INFINITY, 0.f};
    for (int j = 0; ok && j < ntiles; ++j) {
      const int b = j & 1;
      // this warp's keys' scales (keys 64 hk + i of the tile)
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = lane + 32 * u;
        const int64_t kk = (int64_t)j * BN + 64 * hk + i;
        const bool valid = kk < A.T;
        meta[i] = valid ? A.sk[A.t0 + kk] : __float2half(0.f);
        meta[64 + i] = valid ? A.sv[A.t0 + kk] : __float2half(0.f);
      }
      __syncwarp();
      if (!mbar_wait(&B.s_full[b], (j >> 1) & 1, abort, err)) { ok = false; break; }
      tc_fence_after();
      const int64_t rem = A.T - (int64_t)j * BN - 64 * hk;
      const int nk = rem < 0 ? 0 : (rem < 64 ? (int)rem : 64);  // valid keys of this half
      float z[64];
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t s1[32], s2[32];
        tmem_ld32(tmem_lane_addr(tbase, warp, TM_S1 + 64 * b + 32 * c), s1);
        tmem_ld32(tmem_lane_addr(tbase, warp, TM_S2 + 64 * b + 32 * c), s2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sk = __half2float(meta[32 * c + i]);
          const float zz = fmaf(sk, __uint_as_float(s1[i]), zs * __uint_as_float(s2[i]));
          z[32 * c + i] = (32 * c + i < nk) ? zz : -INFINITY;
          mx = fmaxf(mx, z[32 * c + i]);
        }
      }
      // S of this tile is in registers: the buffer may take tile j + 2
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&B.s_free[b]);
      // row maximum over both key halves
      B.xmax[b][hk][row] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.xbar[b]);
      if (!mbar_wait(&B.xbar[b], (j >> 1) & 1, abort, err)) { ok = false; break; }
      const float tmx = fmaxf(B.xmax[b][0][row], B.xmax[b][1][row]);
      float corr = 1.f;
      const bool need = tmx > st.m + kRescaleLog2;  // identical in both halves
      if (need) {
        corr = (st.m == -INFINITY) ? 0.f : ex2(st.m - tmx);
        st.l *= corr;
        st.m = tmx;
      }
      const bool wr = __any_sync(0xffffffffu, need) != 0;
      // the previous tile's value MMAs are done: P / P s_V buffers free, and
      // the accumulators may be rescaled
      // (completion j of pv_done: the prologue was completion 0)
      if (!mbar_wait(&B.pv_done, j & 1, abort, err)) { ok = false; break; }
      if (j > 0 && wr) {
        tc_fence_after();
        rescale_cols(tbase, warp, TM_OT, r / 2 + 64, corr);
      }
      const float m = st.m;
      float ls = 0.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint32_t pp[4], ps[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k0 = 8 * g + 2 * i;
          const float p0 = ex2(z[k0] - m), p1 = ex2(z[k0 + 1] - m);  // exp2(-inf) = 0 past the end
          ls += p0 + p1;
          pp[i] = pack_bf16x2(p0, p1);
          ps[i] = pack_bf16x2(p0 * __half2float(meta[64 + k0]), p1 * __half2float(meta[64 + k0 + 1]));
        }
        st_shared_v4(smem_u32(sP) + sw128_offset(row, 64 * hk + 8 * g, 64), make_uint4(pp[0], pp[1], pp[2], pp[3]));
        st_shared_v4(smem_u32(sPs) + sw128_offset(row, 64 * hk + 8 * g, 64), make_uint4(ps[0], ps[1], ps[2], ps[3]));
      }
      st.l += ls;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&B.p_full);
    }
    // final row sums over both halves, then O~ / l -> bf16 (un-permuted) as the
    // restore's A operand
    if (ok) ok = mbar_wait(&B.pv_done, ntiles & 1, abort, err);  // the last value MMAs
    B.lsum[hk][row] = st.l;
    __syncwarp();
    if (lane == 0) mbar_arrive(&B.lbar);
    if (ok) ok = mbar_wait(&B.lbar, 0, abort, err);
    const float lt = B.lsum[0][row] + B.lsum[1][row];
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    if (ok) {
      tc_fence_after();
      for (int m = 0; m < nm; ++m) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_lane_addr(tbase, warp, TM_OT + 64 * m + 32 * c), v);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            // stored position p holds code (0,4,1,5,2,6,3,7)[p]
            const float *f = reinterpret_cast<const float *>(v + 8 * g);
            const uint4 o = make_uint4(pack_bf16x2(f[0] * inv, f[2] * inv), pack_bf16x2(f[4] * inv, f[6] * inv),
                                       pack_bf16x2(f[1] * inv, f[3] * inv), pack_bf16x2(f[5] * inv, f[7] * inv));
            st_shared_v4(smem_u32(sQt) + sw128_offset(row, 128 * m + 64 * hk + 32 * c + 8 * g, 64), o);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(&B.fin_a);
      if (mbar_wait(&B.fin_done, 0, abort, err)) {
        tc_fence_after();
        // O = O_r + O_c / l for this thread's row and d columns [64 hk, 64 hk + 64)
        const int64_t qrow = q0 + row;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t orr[32], occ[32];
          tmem_ld32(tmem_lane_addr(tbase, warp, TM_S1 + 32 * c), orr);
          tmem_ld32(tmem_lane_addr(tbase, warp, TM_OC + 32 * c), occ);
          if (qrow < A.Tq) {
            float *dst = A.O + (qrow * A.H + h) * DH + 64 * hk + 32 * c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4 *>(dst + i) = make_float4(
                  fmaf(__uint_as_float(occ[i]), inv, __uint_as_float(orr[i])),
                  fmaf(__uint_as_float(occ[i + 1]), inv, __uint_as_float(orr[i + 1])),
                  fmaf(__uint_as_float(occ[i + 2]), inv, __uint_as_float(orr[i + 2])),
                  fmaf(__uint_as_float(occ[i + 3]), inv, __uint_as_float(orr[i + 3])));
          }
        }
        if (hk == 0 && qrow < A.Tq)
          A.L[(int64_t)h * A.Tq + qrow] = lt > 0.f ? (st.m + log2f(lt)) * kLn2 : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // The multicast commits that land in this CTA (kc_empty, s_full, s_last,
  // pv_done, fin_done) have all been waited for by some role above, except
  // kc_empty's last phase, which completes with s_last (same MMAs) and
  // before fin_done; so no commit is in flight into this shared memory.
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc2(tbase, TM_COLS);
  }
}

}  // namespace

size_t tc_low_pair_smem(int r) {
  const int nkb = r / 64, nm = r / 128;
  return (size_t)(nkb + 2 + nkb + 2 + 2 + 2) * kB64 + (size_t)(nm + 1) * kB128 + sizeof(PairBars);
}

bool tc_low_pair_supported(const Codec &ck, const Codec &cv) {
  return ck.prec == PREC_BF16 && ck.d == DH && ck.r == cv.r && ck.r % 128 == 0 && ck.r >= 128 &&
         ck.r <= kMaxR && ck.C <= 256 && cv.C <= 256 && tc_low_pair_smem(ck.r) <= 232448;
}

cudaError_t tc_attend_low_pair(const void *q, int64_t Tq, const Codec &ck, const Codec &cv, const Hist &hk,
                               const Hist &hv, int64_t t0, int64_t T, float tau, Part out, cudaStream_t st,
                               HeadSel hs) {
  if (Tq == 0 || T == 0) return cudaSuccess;
  const int J = ck.H * DH;
  CUtensorMap mq, mdk, mdv;
  if (!make_tmap_bf16_2d(&mq, q, Tq, J, J, 64) || !make_tmap_bf16_2d(&mdk, ck.D, J, ck.r, ck.r, 128) ||
      !make_tmap_bf16_2d(&mdv, cv.D, J, cv.r, cv.r, 64))
    return cudaErrorInvalidValue;
  PairArgs a;
  a.Ck = (const __nv_bfloat16 *)ck.centers;
  a.Cv = (const __nv_bfloat16 *)cv.centers;
  a.idk = hk.ids;
  a.idv = hv.ids;
  a.codk = hk.codes;
  a.codv = hv.codes;
  a.sk = (const __half *)hk.scales;
  a.sv = (const __half *)hv.scales;
  a.t0 = t0;
  a.T = T;
  a.Tq = Tq;
  a.H = ck.H;
  a.r = ck.r;
  a.Ck_n = ck.C;
  a.Cv_n = cv.C;
  a.zscale = tau * kLog2e;
  a.O = out.O;
  a.L = out.LSE;
  a.err = error_word_ptr();
  a.head_map = hs.map;
  const size_t smem = tc_low_pair_smem(ck.r);
  ensure_smem((const void *)tc_low_pair_kernel, (int)smem);
  dim3 grid(2 * (unsigned)((Tq + 127) / 128), (unsigned)(hs.map ? hs.n : ck.H));
  tc_low_pair_kernel<<<grid, 384, smem, st>>>(mq, mdk, mdv, a);
  return cudaGetLastError();
}

}  // namespace nanokv
