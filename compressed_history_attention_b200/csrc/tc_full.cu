// Tensor-core full-dimensional decode-attention (NanoKV Fig. 4(a,b)): the
// history keys and values are decoded on chip,
//     K_hat_t = c_K[a_t] + s_t D_K code_t,   V_hat_t likewise,
// and never written to global memory; then S = tau Q K_hat^T, online softmax,
// O = P V_hat.
//
// A cluster of two CTAs serves two 128-row query tiles of one head.  CTA 0
// decodes K_hat, CTA 1 decodes V_hat, and each writes its decoded bf16 tile
// into the shared memory of both CTAs, so every decode is shared by 256 query
// rows and each CTA keeps a single decoder slice D_h resident.
//
// Roles (12 warps):
//   warp 0      TMEM allocation (otherwise idle)
//   warp 1      TMA (Q tile) and MMA issue: X = codes D_h^T (decode),
//               S = Q K_hat^T, O += P V_hat
//   warps 2,3   unpack: packed INT4 codes, read from global memory, -> bf16
//               operand ring (128 keys x 64 codes per chunk; each warp takes
//               64 of the keys of every chunk)
//   warps 4..7  decode epilogue: X (TMEM, lane = key) * s + center -> bf16 tile
//               in both CTAs' shared memory
//   warps 8..11 softmax, one thread per query row; final O / LSE
// Codes are unpacked in an order permuted within each group of 8; the
// decoder slice is stored with the same permutation, so the contraction over
// the rank index is unchanged.  Every wait is bounded.
//
// The same kernel serves heads deployed at a reduced attention dimension
// d_h in {32, 64, 96} (NanoKV-Fast, Table 6; Fig. 4(d): reduced queries,
// restored outputs).  Its inputs are then the reduced queries U_h^T q and the
// mapped decoder rows U_h^T D_h and centers (W_h for values), so the
// coefficients decode straight into d_h dimensions and every tile, MMA and
// TMEM column range shrinks to d_h; at the end each softmax thread restores
// its normalised row to d dimensions, O = W_h o~, in fp32.
#include "tc_common.cuh"

namespace nanokv {

using namespace sm100;
using namespace tc;

// Optional event trace of the first cluster of head 0 (debug builds with
// -DNANOKV_TRACE only): clock64 stamps per role and key tile.
#ifdef NANOKV_TRACE
__device__ unsigned long long g_full_trace[2][24][128];
#define FULL_TRACE(ev, j)                                                                    \
  do {                                                                                       \
    if (blockIdx.z == 0 && blockIdx.y == 0 && blockIdx.x < 2 && (j) < 128) g_full_trace[rank][ev][j] = clock64(); \
  } while (0)
#else
#define FULL_TRACE(ev, j) \
  do {                    \
  } while (0)
#endif

namespace {

constexpr int DH = 128;
constexpr uint32_t kTile = 128 * 128 * 2;   // [128 x 128] bf16
constexpr uint32_t kChunk = 128 * 64 * 2;   // [128 keys x 64 codes] bf16
constexpr int NRING = 4;  // unpacked code chunks in flight (2 for r > 192: shared memory)
constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
constexpr uint32_t TM_O = 0, TM_S = 128, TM_X = 384, TM_COLS = 512;  // S: two 128-column buffers

struct FullArgs {
  const __nv_bfloat16 *D[2];    // decoders [J, r] (K, V)
  const __nv_bfloat16 *cen[2];  // centers [C, J]
  const uint8_t *ids[2];        // [T_total]
  const uint8_t *codes[2];      // [T_total, r / 2] packed INT4
  const __half *scales[2];      // [T_total]
  int64_t t0, T, Tq;            // branch = history tokens [t0, t0 + T)
  int64_t Tsplit;               // tokens per history split (a multiple of BN); split z = blockIdx.z
  size_t ostride, lstride;      // floats between the partial outputs of consecutive splits
  int H, r, C[2];
  float zscale;
  float *O, *L;
  unsigned *err;
  const int32_t *head_map;      // heads of grid y (nullptr: y is the head)
  const __nv_bfloat16 *W;       // reduced dimension: value maps [H, 128, 128] (restore)
};

struct FullBars {
  uint64_t q_full;
  uint64_t ring_full[NRING], ring_empty[NRING];
  uint64_t x_full, x_empty;
  uint64_t kh_full, vh_full, kh_empty, vh_empty;
  uint64_t s_full[2], p_full[2], pv_done[2];  // pv_done[b]: P*V of the tiles using S buffer b
  uint32_t tmem_base;
  int abort;
};

// 8 packed INT4 codes (one 32-bit word, code i in bits [4i, 4i+4)) -> 8 bf16
// in the order (n0,n4), (n1,n5), (n2,n6), (n3,n7): position p of the group
// holds code (0,4,1,5,2,6,3,7)[p]
// kLarge (codecs with r > 192 or C > 64): the branch's centers are read from
// global memory (L2) by the epilogue instead of being staged in shared
// memory, and the code ring has 2 slots, so that a resident decoder slice of
// up to r = 384 fits.
//
// DHR: attention dimension of the launch (128, or a reduced d_h of 32, 64 or
// 96).  Q and decoded tiles are [128 x DHR] in 64-column blocks (NAT of
// them); the decoder slice holds DHR rows.
template <int DHR>
struct FullDims {
  static constexpr int NAT = (DHR + 63) / 64;
  static constexpr uint32_t kTileR = NAT * (kTile / 2);  // bytes of a Q / decoded tile
  static constexpr uint32_t kDChunk = DHR * 128;          // decoder bytes per 64-wide rank block
  static constexpr uint32_t IDEC = idesc_bf16(128, DHR, false, false);
  static constexpr uint32_t IPV = idesc_bf16(128, DHR, false, true);
};

template <bool kLarge, int DHR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    tc_full_kernel(const __grid_constant__ CUtensorMap tmQ, const FullArgs A) {
  using F = FullDims<DHR>;
  constexpr int NAT = F::NAT;
  constexpr uint32_t kTileR = F::kTileR;
  extern __shared__ uint8_t smraw[];
  uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  const int nrb = A.r / 64;  // 64-wide rank blocks
  uint8_t *sQ = sm;
  uint8_t *sD = sQ + kTileR;
  uint8_t *sRing = sD + nrb * F::kDChunk;
  constexpr bool kCenGlobal = kLarge;
  constexpr int nring = kLarge ? 2 : NRING;
  uint8_t *sKh = sRing + nring * kChunk;
  uint8_t *sVh = sKh + kTileR;
  uint8_t *sCen = sVh + kTileR;  // this CTA's branch centers, head slice [C][DHR] bf16, 256-byte rows
  __shared__ FullBars B;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: decodes K, 1: decodes V
  const uint32_t peer = rank ^ 1u;
  const int h = A.head_map ? A.head_map[blockIdx.y] : (int)blockIdx.y;
  const int64_t q0 = (int64_t)blockIdx.x * BM;
  // this CTA's share of the history: split blockIdx.z, tokens [t0, t0 + T)
  const int64_t tb = (int64_t)blockIdx.z * A.Tsplit;
  const int64_t t0 = A.t0 + tb;
  const int64_t T = (A.T - tb) < A.Tsplit ? (A.T - tb) : A.Tsplit;
  const int ntiles = (int)((T + BN - 1) / BN);
  const int nchunk = ntiles * nrb;
  const int J = A.H * DH;
  volatile int *abort = &B.abort;
  unsigned *err = A.err;

  if (threadIdx.x == 0) {
    mbar_init(&B.q_full, 1);
    for (int i = 0; i < nring; ++i) { mbar_init(&B.ring_full[i], 2); mbar_init(&B.ring_empty[i], 1); }
    mbar_init(&B.x_full, 1);
    mbar_init(&B.x_empty, 4);  // one arrive per epilogue warp once its last X load is done
    // decoded-tile barriers: in the decoding CTA one arrive per epilogue
    // warp; in the receiving CTA one expect_tx arrive, by its own MMA
    // thread, that arms each phase for the bytes of the decoder's bulk copies
    mbar_init(&B.kh_full, rank == 0 ? 4 : 1);
    mbar_init(&B.vh_full, rank == 1 ? 4 : 1);
    mbar_init(&B.kh_empty, 2);
    mbar_init(&B.vh_empty, 2);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.p_full[i], 4);
      mbar_init(&B.pv_done[i], 1);
    }
    B.abort = 0;
    // phase 0 of the barrier of the tile this CTA receives
    mbar_arrive_expect_tx(rank == 1 ? &B.kh_full : &B.vh_full, kTileR);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&B.tmem_base, TM_COLS);
    tmem_relinquish();
  }
  // decoder slice of this CTA's branch, rows h*128.. of D [J, r], permuted
  // within groups of 8 like the unpacked codes (K-major 128B-swizzled), and
  // the head slice of its centers, 16-byte chunk k of row a stored at chunk
  // (k ^ (a & 15)) so that rows read together spread over the banks.  All
  // threads stage them with several 16-byte loads in flight each.
  {
    const __nv_bfloat16 *Dsrc = A.D[rank] + (size_t)h * DH * A.r;
    const int gpr = A.r / 8;  // 8-element groups per row
    const int groups = DHR * gpr;
    constexpr int U = 8;
    for (int g0 = threadIdx.x; g0 < groups; g0 += U * 384) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int gidx = g0 + u * 384;
        if (gidx < groups) v[u] = *reinterpret_cast<const uint4 *>(Dsrc + (size_t)(gidx / gpr) * A.r + 8 * (gidx % gpr));
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int gidx = g0 + u * 384;
        if (gidx < groups) {
          // element order (0,4,1,5,2,6,3,7): 16-bit halves of the source words
          const uint4 o = make_uint4(__byte_perm(v[u].x, v[u].z, 0x5410), __byte_perm(v[u].x, v[u].z, 0x7632),
                                     __byte_perm(v[u].y, v[u].w, 0x5410), __byte_perm(v[u].y, v[u].w, 0x7632));
          *reinterpret_cast<uint4 *>(sD + sw128_offset(gidx / gpr, 8 * (gidx % gpr), DHR)) = o;
        }
      }
    }
    const int C = kCenGlobal ? 0 : A.C[rank];  // nothing to stage when centers are read from L2
    const __nv_bfloat16 *cen = A.cen[rank] + (size_t)h * DH;
    constexpr int CPR = DHR / 8;  // 16-byte chunks per center row
    for (int i0 = threadIdx.x; i0 < C * CPR; i0 += 4 * 384) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 384;
        if (i < C * CPR) v[u] = *reinterpret_cast<const uint4 *>(cen + (size_t)(i / CPR) * J + 8 * (i % CPR));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 384;
        if (i < C * CPR) {
          const int a = i / CPR, k = i % CPR;
          *reinterpret_cast<uint4 *>(sCen + a * 256 + ((k ^ (a & 15)) << 4)) = v[u];
        }
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tbase = B.tmem_base;
  pdl_launch_dependents();

  if (warp == 1) {
    // ---------------- Q load and MMA issuer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      mbar_arrive_expect_tx(&B.q_full, kTileR);
#pragma unroll
      for (int c = 0; c < NAT; ++c) tma_load_2d(sQ + c * (kTile / 2), &tmQ, h * DH + 64 * c, (int)q0, &B.q_full);
      const uint32_t aQ = smem_u32(sQ), aD = smem_u32(sD), aR = smem_u32(sRing);
      const uint32_t aK = smem_u32(sKh), aV = smem_u32(sVh);
      bool ok = mbar_wait(&B.q_full, 0, abort, err);
      // Three independent MMA streams, each issued as soon as its inputs are
      // ready (polled with non-blocking tests), so that none waits behind
      // another: decode chunks (X = codes D_h^T), scores S_j = Q K_hat_j^T,
      // values O += P_j V_hat_j.
      int jd = 0, cb = 0, cc = 0;  // decode: tile, rank block within it, chunk counter
      int js = 0, jv = 0;          // next scores / values tile
      uint64_t t_last = globaltimer();
      while (ok && jv < ntiles) {
        bool progress = false;
        // ---- decode stream
        if (jd < ntiles && (cb > 0 || jd == 0 || mbar_test(&B.x_empty, (jd - 1) & 1))) {
          const int slot = cc % nring;
          if (mbar_test(&B.ring_full[slot], (cc / nring) & 1)) {
            if (cb == 0) FULL_TRACE(0, jd);
            tc_fence_after();
            const uint32_t a = aR + slot * kChunk, b = aD + cb * F::kDChunk;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_ss(tbase + TM_X, sdesc_sw128(a + 32 * k, 16, 1024), sdesc_sw128(b + 32 * k, 16, 1024), F::IDEC,
                     (cb > 0 || k > 0));
            mma_commit(&B.ring_empty[slot]);
            ++cc;
            if (++cb == nrb) {
              mma_commit(&B.x_full);
              FULL_TRACE(1, jd);
              cb = 0;
              ++jd;
            }
            progress = true;
          }
        }
        // ---- scores stream (the S buffer of tile js last held P of js - 2)
        if (js < ntiles && mbar_test_cluster(&B.kh_full, js & 1) &&
            (js < 2 || mbar_test(&B.pv_done[js & 1], ((js - 2) >> 1) & 1))) {
          FULL_TRACE(2, js);
          // the K_hat receiver arms the next phase (its bytes can only come
          // after this tile's scores are done in both CTAs)
          if (rank == 1 && js + 1 < ntiles) mbar_arrive_expect_tx(&B.kh_full, kTileR);
          tc_fence_after();
          const uint32_t dS = tbase + TM_S + (js & 1) * 128;
#pragma unroll
          for (int ks = 0; ks < DHR / 16; ++ks) {
            const uint32_t off = (ks >> 2) * (kTile / 2) + (ks & 3) * 32;
            mma_ss(dS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024), IDESC_S, ks > 0);
          }
          mma_commit(&B.s_full[js & 1]);
          mma_commit_mc(&B.kh_empty, 0x1);  // K_hat consumed here: tell the K decoder (CTA 0)
          ++js;
          progress = true;
        }
        // ---- values stream
        if (jv < js && mbar_test(&B.p_full[jv & 1], (jv >> 1) & 1) && mbar_test_cluster(&B.vh_full, jv & 1)) {
          FULL_TRACE(3, jv);
          if (rank == 0 && jv + 1 < ntiles) mbar_arrive_expect_tx(&B.vh_full, kTileR);
          tc_fence_after();
          const uint32_t sP = tbase + TM_S + (jv & 1) * 128;
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_ts(tbase + TM_O, sP + ks * 8, sdesc_sw128(aV + ks * 2048, kTile / 2, 1024), F::IPV,
                   (jv > 0 || ks > 0));
          mma_commit(&B.pv_done[jv & 1]);
          mma_commit_mc(&B.vh_empty, 0x2);  // V_hat consumed: tell the V decoder (CTA 1)
          ++jv;
          progress = true;
        }
        // no sleep between polls: the time to notice a completed barrier is
        // on every chain through this thread
        if (progress) {
          t_last = globaltimer();
        } else {
          if (*abort) break;
          if (globaltimer() - t_last > kWaitLimitNs) {
            *abort = 1;
            atomicOr(err, ERRW_TIMEOUT);
            break;
          }
        }
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------- unpack: packed codes -> ring (bf16, K-major SW128) ----------------
    // Each thread takes keys kb + lane and kb + 32 + lane of every chunk and
    // reads their 32 code bytes straight from global memory, one chunk ahead.
    // (The codes go to registers, not through a shared staging buffer that a
    // copy engine would refill while these loads might still be in flight.)
    const uint8_t *codes = A.codes[rank];
    const int64_t rowb = A.r / 2;        // packed bytes per token
    const int kb = (warp - 2) * 64;
    auto load = [&](int c, uint4(&v)[4]) {
      const int j = c / nrb, cb = c % nrb;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        int64_t t = (int64_t)j * BN + kb + lane + 32 * i;
        t = t < T ? t : T - 1;  // keys past the end: any valid row (masked later)
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + (t0 + t) * rowb + cb * 32);
        v[2 * i] = __ldg(src);
        v[2 * i + 1] = __ldg(src + 1);
      }
    };
    uint4 cur[4], nxt[4], nx2[4], nx3[4];
    load(0, cur);
    if (1 < nchunk) load(1, nxt);
    if (2 < nchunk) load(2, nx2);
    for (int c = 0; c < nchunk; ++c) {
      if (c + 3 < nchunk) load(c + 3, nx3);
      const int rs = c % nring, cb = c % nrb;
      if (warp == 2 && lane == 0 && cb == 0) FULL_TRACE(9, c / nrb);
      if (warp == 2 && lane == 0 && cb == 1) FULL_TRACE(17, c / nrb);
      if (c >= nring && !mbar_wait(&B.ring_empty[rs], ((c / nring) - 1) & 1, abort, err)) break;
      if (warp == 2 && lane == 0 && cb == 0) FULL_TRACE(10, c / nrb);
      if (warp == 2 && lane == 0 && cb == 1) FULL_TRACE(18, c / nrb);
      const uint32_t dst = smem_u32(sRing + rs * kChunk);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t w[8] = {cur[2 * i].x,     cur[2 * i].y,     cur[2 * i].z,     cur[2 * i].w,
                               cur[2 * i + 1].x, cur[2 * i + 1].y, cur[2 * i + 1].z, cur[2 * i + 1].w};
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          st_shared_v4(dst + sw128_offset(kb + lane + 32 * i, 8 * g, 128), unpack8(w[g]));
          if (i == 0 && g == 0 && warp == 2 && lane == 0 && cb == 1) FULL_TRACE(21, c / nrb);
        }
      }
      if (warp == 2 && lane == 0 && cb == 1) FULL_TRACE(19, c / nrb);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.ring_full[rs]);
      if (warp == 2 && lane == 0 && cb == nrb - 1) FULL_TRACE(11, c / nrb);
      if (warp == 2 && lane == 0 && cb == 1) FULL_TRACE(20, c / nrb);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        cur[k] = nxt[k];
        nxt[k] = nx2[k];
        nx2[k] = nx3[k];
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- decode epilogue (thread = key) ----------------
    const int t = (warp - 4) * 32 + lane;
    const int C = A.C[rank];
    uint8_t *dstL = rank == 0 ? sKh : sVh;
    const uint32_t dst_local = smem_u32(dstL);
    const uint32_t dst_remote = mapa(dst_local, peer);
    uint64_t *full_bar = rank == 0 ? &B.kh_full : &B.vh_full;
    uint64_t *empty_bar = rank == 0 ? &B.kh_empty : &B.vh_empty;
    const uint32_t full_remote = mapa(smem_u32(full_bar), peer);
    auto key_meta = [&](int j, int &a, float &s) {
      const int64_t tt = t0 + (int64_t)j * BN + t;
      const bool valid = (int64_t)j * BN + t < T;
      a = valid ? (int)A.ids[rank][tt] : 0;
      a = a < C ? a : C - 1;
      s = valid ? __half2float(A.scales[rank][tt]) : 0.f;
    };
    int a_next;
    float s_next;
    key_meta(0, a_next, s_next);
    for (int j = 0; j < ntiles; ++j) {
      const int a = a_next;
      const float s = s_next;
      if (j + 1 < ntiles) key_meta(j + 1, a_next, s_next);
      const uint8_t *crow = sCen + a * 256;
      const int sw = a & 15;
      uint32_t o[DHR / 2];
      if constexpr (kCenGlobal) {
        // the key's center row (known a tile ahead) from L2, into the output
        // registers, before X is ready: o = c + s x is then formed in place
        const uint4 *src = reinterpret_cast<const uint4 *>(A.cen[rank] + (size_t)a * J + (size_t)h * DH);
#pragma unroll
        for (int g = 0; g < DHR / 8; ++g) {
          const uint4 cv = __ldg(src + g);
          o[4 * g] = cv.x;
          o[4 * g + 1] = cv.y;
          o[4 * g + 2] = cv.z;
          o[4 * g + 3] = cv.w;
        }
      }
      if (!mbar_wait(&B.x_full, j & 1, abort, err)) break;
      if (t == 0) FULL_TRACE(4, j);
      tc_fence_after();
      // K_hat = c + s x in packed bf16x2: x rounded to bf16, one fused
      // multiply-add per pair, one rounding of the result.  The whole row is
      // computed into registers and X released before the destination
      // buffer is waited for, so the next decode overlaps the hand-off.
      const __nv_bfloat162 s2 = __floats2bfloat162_rn(s, s);
#pragma unroll
      for (int c = 0; c < DHR / 32; ++c) {
        uint32_t x[32];
        tmem_ld32(tmem_lane_addr(tbase, warp, TM_X + 32 * c), x);
        if (c == DHR / 32 - 1) {
          // X is no longer read by this warp: let the next decode start now
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&B.x_empty);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t cw[4];
          if constexpr (kCenGlobal) {
#pragma unroll
            for (int i = 0; i < 4; ++i) cw[i] = o[16 * c + 4 * g + i];
          } else {
            const uint4 cv = *reinterpret_cast<const uint4 *>(crow + (((4 * c + g) ^ sw) << 4));
            cw[0] = cv.x;
            cw[1] = cv.y;
            cw[2] = cv.z;
            cw[3] = cv.w;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t xp = pack_bf16x2(__uint_as_float(x[8 * g + 2 * i]), __uint_as_float(x[8 * g + 2 * i + 1]));
            const __nv_bfloat162 r = __hfma2(s2, *reinterpret_cast<const __nv_bfloat162 *>(&xp),
                                             *reinterpret_cast<const __nv_bfloat162 *>(&cw[i]));
            o[16 * c + 4 * g + i] = *reinterpret_cast<const uint32_t *>(&r);
          }
        }
      }
      if (t == 0) FULL_TRACE(22, j);
      // the previous tile in this buffer was consumed by both CTAs (and the
      // bulk copy that carried it to the peer had completed before that)
      if (j > 0 && !mbar_wait_cluster(empty_bar, (j - 1) & 1, abort, err)) break;
      if (t == 0) FULL_TRACE(5, j);
#pragma unroll
      for (int c = 0; c < NAT; ++c) {
        constexpr int G = DHR >= 64 ? 8 : DHR / 8;  // 8-column groups of a block (the last one may hold fewer)
#pragma unroll
        for (int g = 0; g < G; ++g)
          if (64 * c + 8 * g < DHR)
            st_shared_v4(dst_local + sw128_offset(t, 64 * c + 8 * g, 128),
                         make_uint4(o[32 * c + 4 * g], o[32 * c + 4 * g + 1], o[32 * c + 4 * g + 2],
                                    o[32 * c + 4 * g + 3]));
        // columns [64c, 64c + 64) of every key form one 16 KB block of the
        // tile, and this warp's 32 key rows of it are contiguous: each warp
        // hands its rows to the peer as soon as it has stored them
        if (t == 0 && c == 0) FULL_TRACE(12, j);
        fence_proxy_async_smem();  // read by this CTA's MMA and by the bulk copy
        __syncwarp();
        if (lane == 0) {
          const uint32_t off = c * (kTile / 2) + (uint32_t)(warp - 4) * 32 * 128;
          bulk_s2cluster(dst_remote + off, dstL + off, 32 * 128, full_remote);
        }
      }
      if (lane == 0) mbar_arrive(full_bar);  // the local MMA may read this warp's rows
      if (t == 0) FULL_TRACE(6, j);
    }
  } else if (warp >= 8) {
    // ---------------- softmax (thread = query row) ----------------
    const int row = (warp - 8) * 32 + lane;
    RowState st{-INFINITY, 0.f};
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!mbar_wait(&B.s_full[j & 1], (j >> 1) & 1, abort, err)) { ok = false; break; }
      if (row == 0) FULL_TRACE(7, j);
      tc_fence_after();
      const int64_t rem = T - (int64_t)j * BN;
      const int nk = rem < BN ? (int)rem : BN;
      bool wr;
#ifdef NANOKV_TRACE
      const int tj = (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && row == 0) ? j : -1;
#else
      const int tj = -1;
#endif
      const float corr = softmax_tile(tbase, warp, TM_S + (j & 1) * 128, nk, A.zscale, st, wr, tj);
      if (j > 0 && wr) {
        if (!mbar_wait(&B.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort, err)) { ok = false; break; }
        tc_fence_after();
        rescale_o(tbase, warp, TM_O, corr, DHR / 16);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_full[j & 1]);
      if (row == 0) FULL_TRACE(8, j);
    }
    // the value MMAs may trail the softmax by two tiles: wait for the last two
    // phases in order so that a parity can never be mistaken for an older one
    if (ok && ntiles >= 2) ok = mbar_wait(&B.pv_done[(ntiles - 2) & 1], ((ntiles - 2) >> 1) & 1, abort, err);
    if (ok && mbar_wait(&B.pv_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, abort, err)) {
      tc_fence_after();
      if constexpr (DHR == DH)
        write_row(tbase, warp, TM_O, st, q0 + row, A.Tq, h, A.H, A.O + blockIdx.z * A.ostride,
                  A.L + blockIdx.z * A.lstride);
      else
        write_row_restored<DHR>(tbase, warp, TM_O, st, q0 + row, A.Tq, h, A.H, A.W + (size_t)h * DH * DH,
                                A.O + blockIdx.z * A.ostride, A.L + blockIdx.z * A.lstride);
    }
  }
  tc_fence_before();
  __syncthreads();
  // the peer's last consumer signals (multicast commits) must land before this
  // CTA's shared memory goes away; after the block barrier the epilogue has
  // waited every earlier phase, so this wait cannot see a stale parity
  if (threadIdx.x == 0 && !*abort) {
    if (rank == 0) mbar_wait_cluster(&B.kh_empty, (ntiles - 1) & 1, nullptr, nullptr);
    else mbar_wait_cluster(&B.vh_empty, (ntiles - 1) & 1, nullptr, nullptr);
  }
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
  pdl_wait_prior();
}

}  // namespace

static bool full_large(int r, int C) { return r > 192 || C > 64; }

static size_t tc_full_smem(int r, int C, int dhr = DH) {
  const bool large = full_large(r, C);
  const size_t tile = (size_t)((dhr + 63) / 64) * (kTile / 2);
  return 3 * tile + (size_t)(r / 64) * dhr * 128 + (size_t)(large ? 2 : NRING) * kChunk +
         (large ? 0 : (size_t)C * 256) + 1024;
}

bool tc_full_supported(const Codec &ck, const Codec &cv) {
  // shared memory: Q, the resident decoder slice (r / 64 blocks), the code
  // ring, two decoded tiles and, for at most 64 centers, the center slice
  const int C = ck.C > cv.C ? ck.C : cv.C;
  return ck.prec == PREC_BF16 && ck.d == DH && ck.r == cv.r && ck.r % 64 == 0 && ck.r <= 384 &&
         C <= 256 && tc_full_smem(ck.r, C) <= 232448;
}

bool tc_reduced_dim_ok(int d_h) { return d_h == 32 || d_h == 64 || d_h == 96; }

// Largest number of two-CTA clusters of the full-dim kernel that can be
// resident at once on the current device (cached per device).
static int full_cluster_capacity() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] > 0) return cached[dev];
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int cap = sms / 2;
  const size_t smem = tc_full_smem(192, 64);
  if (ensure_smem((const void *)tc_full_kernel<false, DH>, (int)smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(384);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (const void *)tc_full_kernel<false, DH>, &cfg) == cudaSuccess && n > 0)
      cap = n;
  }
  cudaGetLastError();
  cached[dev] = cap > 0 ? cap : 1;
  return cached[dev];
}

int tc_full_splits(int64_t Tq, int H, int d, int64_t T) {
  // Cost model in microseconds: the launch runs ceil(units * ns / capacity)
  // waves of clusters, each cluster ~3.3 us per 128-key tile plus ~6 tiles of
  // fixed cost (staging, pipeline fill and drain); every extra split adds a
  // [Tq, H, d] fp32 partial written here and read by the merge, counted
  // twice over because the other branches' kernels, which run alongside,
  // fill part of a ragged last wave anyway.  (Measured on the full-size
  // workloads: 2 splits best at 110 key tiles, 1 at 37.)
  if (T <= 0 || Tq <= 0) return 1;
  const int64_t ntiles = (T + BN - 1) / BN;
  const int64_t units = (int64_t)H * ((((Tq + BM - 1) / BM) + 1) / 2);
  const int64_t cap = full_cluster_capacity();
  if (cap <= 0) return 1;
  const double part_us = 4.0 * (double)Tq * H * d * 4.0 / 6.0e6;
  int best = 1;
  double best_cost = 1e300;
  for (int ns = 1; ns <= kMaxFullSplits && ns <= ntiles; ++ns) {
    const int64_t per = (ntiles + ns - 1) / ns;
    if ((ntiles + per - 1) / per != ns) continue;  // some split would be empty
    const int64_t waves = (units * ns + cap - 1) / cap;
    const double cost = (double)waves * ((double)per + 6.0) * 3.3 + (ns - 1) * part_us;
    if (cost < best_cost * 0.99) {
      best_cost = cost;
      best = ns;
    }
  }
  return best;
}

template <int DHR>
static cudaError_t launch_full(const CUtensorMap &mq, const FullArgs &a, dim3 grid, bool large, size_t smem,
                               cudaStream_t st, bool pdl) {
  const void *fn = large ? (const void *)tc_full_kernel<true, DHR> : (const void *)tc_full_kernel<false, DHR>;
  cudaError_t e = ensure_smem(fn, (int)smem);
  if (e != cudaSuccess) return e;
  return large ? launch_k(tc_full_kernel<true, DHR>, grid, dim3(384), smem, st, pdl, mq, a)
               : launch_k(tc_full_kernel<false, DHR>, grid, dim3(384), smem, st, pdl, mq, a);
}

static cudaError_t attend_full_dim(int dhr, const void *q, int64_t Tq, const Codec &ck, const Codec &cv,
                                   const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau, Part out,
                                   int nsplit, size_t ostride, size_t lstride, cudaStream_t st, bool pdl, HeadSel hs,
                                   const void *W) {
  if (Tq == 0 || T == 0) return cudaSuccess;
  const int64_t ntiles = (T + BN - 1) / BN;
  if (nsplit < 1 || nsplit > ntiles) return cudaErrorInvalidValue;
  const int J = ck.H * DH;
  CUtensorMap mq;
  if (!make_tmap_bf16_2d(&mq, q, Tq, J, J, 128)) return cudaErrorInvalidValue;
  FullArgs a;
  a.D[0] = (const __nv_bfloat16 *)ck.D;
  a.D[1] = (const __nv_bfloat16 *)cv.D;
  a.cen[0] = (const __nv_bfloat16 *)ck.centers;
  a.cen[1] = (const __nv_bfloat16 *)cv.centers;
  a.ids[0] = hk.ids;
  a.ids[1] = hv.ids;
  a.codes[0] = hk.codes;
  a.codes[1] = hv.codes;
  a.scales[0] = (const __half *)hk.scales;
  a.scales[1] = (const __half *)hv.scales;
  a.t0 = t0;
  a.T = T;
  a.Tsplit = ((ntiles + nsplit - 1) / nsplit) * BN;
  a.ostride = ostride;
  a.lstride = lstride;
  a.Tq = Tq;
  a.H = ck.H;
  a.r = ck.r;
  a.C[0] = ck.C;
  a.C[1] = cv.C;
  a.zscale = tau * kLog2e;
  a.O = out.O;
  a.L = out.LSE;
  a.err = error_word_ptr();
  a.head_map = hs.map;
  a.W = (const __nv_bfloat16 *)W;
  const int Cmax = ck.C > cv.C ? ck.C : cv.C;
  const bool large = full_large(ck.r, Cmax);
  const size_t smem = tc_full_smem(ck.r, Cmax, dhr);
  if (smem > 232448) return cudaErrorInvalidConfiguration;
  const unsigned qt = (unsigned)((Tq + BM - 1) / BM);
  // every split must get at least one key tile (the caller merges nsplit partials)
  if ((T + a.Tsplit - 1) / a.Tsplit != nsplit) return cudaErrorInvalidValue;
  dim3 grid((qt + 1) & ~1u, (unsigned)(hs.map ? hs.n : ck.H), (unsigned)nsplit);
  switch (dhr) {
    case 32: return launch_full<32>(mq, a, grid, large, smem, st, pdl);
    case 64: return launch_full<64>(mq, a, grid, large, smem, st, pdl);
    case 96: return launch_full<96>(mq, a, grid, large, smem, st, pdl);
    case DH: return launch_full<DH>(mq, a, grid, large, smem, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t tc_attend_full(const void *q, int64_t Tq, const Codec &ck, const Codec &cv, const Hist &hk,
                           const Hist &hv, int64_t t0, int64_t T, float tau, Part out, int nsplit, size_t ostride,
                           size_t lstride, cudaStream_t st, bool pdl, HeadSel hs) {
  return attend_full_dim(DH, q, Tq, ck, cv, hk, hv, t0, T, tau, out, nsplit, ostride, lstride, st, pdl, hs, nullptr);
}

cudaError_t tc_attend_reduced(int d_h, const void *q_red, int64_t Tq, const Codec &ck_red, const Codec &cv_red,
                              const void *W, const Hist &hk, const Hist &hv, int64_t t0, int64_t T, float tau,
                              Part out, cudaStream_t st, HeadSel hs) {
  if (!tc_reduced_dim_ok(d_h) || !W) return cudaErrorInvalidValue;
  return attend_full_dim(d_h, q_red, Tq, ck_red, cv_red, hk, hv, t0, T, tau, out, 1, 0, 0, st, false, hs, W);
}

#ifdef NANOKV_TRACE
extern "C" int nanokv_debug_full_trace(void *host, size_t bytes) {
  if (bytes < sizeof(g_full_trace) + sizeof(g_softmax_trace)) return -1;
  if (cudaMemcpyFromSymbol(host, g_full_trace, sizeof(g_full_trace)) != cudaSuccess) return -3;
  return cudaMemcpyFromSymbol((char *)host + sizeof(g_full_trace), g_softmax_trace, sizeof(g_softmax_trace)) ==
                 cudaSuccess
             ? 0
             : -3;
}
#endif

}  // namespace nanokv
