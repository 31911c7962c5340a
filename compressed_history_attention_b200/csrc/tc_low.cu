// Tensor-core mixed-dimensional attention over the history a fixed policy
// routes to low dimension (NanoKV-Fast; abstract: reuse the stored
// coefficients; Fig. 4(d): reduce the queries, restore the output dimension).
// Per head h, with D_h the head's rows of D and c_{j,h} its slice of center j:
//   prologue   Q~ = Q D_{K,h}  [128 x r],  QC = Q C_{K,h}^T  [128 x C]   (MMA)
//   per tile   S' = Q~ codes_K^T                                      (MMA)
//              z  = tau (s_K S' + QC[a_K])          (softmax warps, log2 units)
//              O~ += (P * s_V) codes_V,   P_C += P onehot(a_V)        (MMA)
//   epilogue   O  = (O~ D_{V,h}^T + P_C C_{V,h}) / l                  (MMA)
// P and P * s_V are written back to TMEM as bf16, interleaved per 32 keys.
// Codes are unpacked in the order (0,4,1,5,2,6,3,7) within each group of 8;
// Q~ is stored with the same order and O~ is un-permuted before the restore.
//   warp 0      TMA: Q, D_{K,h}, C_{K,h}; later D_{V,h}, C_{V,h}
//   warp 1      MMA issuer
//   warps 2,3   key-side unpack: K codes, center ids and scales (two keys a thread)
//   warps 4..7  value-side unpack: thread = key; V codes, one-hot of a_V
//   warps 8..11 softmax, one thread per query row; prologue/epilogue stores
#include "tc_common.cuh"

namespace nanokv {

using namespace sm100;
using namespace tc;

// Optional event trace of the first CTA (debug builds with -DNANOKV_TRACE only):
// clock64 stamps per role and key tile.
#ifdef NANOKV_TRACE
__device__ unsigned long long g_low_trace[12][128];
#define LOW_TRACE(ev, j)                                                                    \
  do {                                                                                      \
    if (blockIdx.x == 0 && blockIdx.y == 0 && (j) < 128) g_low_trace[ev][j] = clock64();    \
  } while (0)
#else
#define LOW_TRACE(ev, j) \
  do {                   \
  } while (0)
#endif

namespace {

constexpr int DH = 128;
constexpr uint32_t kBlk = 128 * 64 * 2;  // [128 rows x 64] bf16 block
constexpr uint32_t TM_OT = 0, TM_S0 = 256, TM_COLS = 512;
constexpr int kMaxCodeWords = 6;  // uint4 words of packed codes per key (r <= 192)

struct LowArgs {
  const __nv_bfloat16 *Dk, *Dv;   // decoders [J, r]
  const __nv_bfloat16 *Ck, *Cv;   // centers [C, J]
  const uint8_t *idk, *idv;       // [T]
  const uint8_t *codk, *codv;     // [T, r/2]
  const __half *sk, *sv;          // [T]
  int64_t t0, T, Tq;
  int H, r, C;
  float zscale;
  float *O, *L;
  unsigned *err;
  const int32_t *head_map;  // heads of grid y (nullptr: y is the head)
};


struct LowBars {
  uint64_t pro_full, pro_done, qt_ready;
  uint64_t kc_full, kc_empty, vc_full, v_empty;
  uint64_t s_full[2], p_full[2], info_full[2], pv_done[2], last_done;  // pv_done[b]: P*V of the tiles using S buffer b
  uint64_t fin_a, fin_b, fin_done;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(384, 1)
    tc_low_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDk,
                  const __grid_constant__ CUtensorMap tmCk, const __grid_constant__ CUtensorMap tmDv,
                  const __grid_constant__ CUtensorMap tmCv, const LowArgs A) {
  extern __shared__ uint8_t smraw[];
  uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  const int r = A.r, C = A.C;
  const int nrb = r / 64;
  uint8_t *sQt = sm;                           // [128 x r] K-major (persistent)
  uint8_t *sKc = sQt + nrb * kBlk;             // [128 keys x r] K-major
  uint8_t *sVc = sKc + nrb * kBlk;             // [128 keys x r] (MN-major use)
  uint8_t *sOH = sVc + nrb * kBlk;             // [128 keys x C] one-hot
  float *sQC = (float *)(sOH + kBlk);          // [128][C + 1]
  // per-key info of the two tiles in flight, as arrays (16-byte aligned) so
  // that the softmax reads four keys' values with one broadcast load
  int *kAK = (int *)(sQC + 128 * (C + 1));  // [2][128] key center id
  float *kSK = (float *)(kAK + 2 * 128);     // [2][128] key scale
  float *kSV = kSK + 2 * 128;                // [2][128] value scale
  // prologue aliases (inside sKc .. sOH)
  uint8_t *sQ = sKc;                           // [128 x 128] K-major
  uint8_t *sDk = sKc + 2 * kBlk;               // D_{K,h} [128 d x r] (MN-major use)
  uint8_t *sCk = sDk + nrb * kBlk;             // C_{K,h} [C x 128] K-major (2 blocks of C*128 B)
  // epilogue aliases
  uint8_t *sAo = sKc;                          // O~ / l  [128 x r] K-major
  uint8_t *sAp = sOH;                          // P_C / l [128 x C] K-major
  uint8_t *sDv = sVc;                          // D_{V,h} [128 d x r] K-major
  uint8_t *sCv = sQt;                          // C_{V,h} [C x 128] (MN-major use)
  __shared__ LowBars B;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = A.head_map ? A.head_map[blockIdx.y] : (int)blockIdx.y;
  const int64_t q0 = (int64_t)blockIdx.x * BM;
  const int ntiles = (int)((A.T + BN - 1) / BN);
  volatile int *abort = &B.abort;
  unsigned *err = A.err;
  const uint32_t cblk = (uint32_t)C * 128;  // bytes of one [C rows x 64] block

  if (threadIdx.x == 0) {
    mbar_init(&B.pro_full, 1);
    mbar_init(&B.pro_done, 1);
    mbar_init(&B.qt_ready, 4);
    mbar_init(&B.kc_full, 2);  // the two key-side unpack warps
    mbar_init(&B.kc_empty, 1);
    mbar_init(&B.vc_full, 4);
    mbar_init(&B.v_empty, 1);
    mbar_init(&B.s_full[0], 1);
    mbar_init(&B.s_full[1], 1);
    mbar_init(&B.p_full[0], 4);
    mbar_init(&B.p_full[1], 4);
    mbar_init(&B.info_full[0], 2);
    mbar_init(&B.info_full[1], 2);
    mbar_init(&B.pv_done[0], 1);
    mbar_init(&B.pv_done[1], 1);
    mbar_init(&B.last_done, 1);
    mbar_init(&B.fin_a, 4);
    mbar_init(&B.fin_b, 1);
    mbar_init(&B.fin_done, 1);
    B.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&B.tmem_base, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = B.tmem_base;
  pdl_launch_dependents();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      mbar_arrive_expect_tx(&B.pro_full, 2 * kBlk + nrb * kBlk + 2 * cblk);
      tma_load_2d(sQ, &tmQ, h * DH, (int)q0, &B.pro_full);
      tma_load_2d(sQ + kBlk, &tmQ, h * DH + 64, (int)q0, &B.pro_full);
      for (int b = 0; b < nrb; ++b) tma_load_2d(sDk + b * kBlk, &tmDk, 64 * b, h * DH, &B.pro_full);
      for (int b = 0; b < 2; ++b) tma_load_2d(sCk + b * cblk, &tmCk, h * DH + 64 * b, 0, &B.pro_full);
      bool ok = mbar_wait(&B.pro_full, 0, abort, err);
      // restore operands once every tile's MMAs are done
      if (ok && mbar_wait(&B.last_done, 0, abort, err)) {
        mbar_arrive_expect_tx(&B.fin_b, nrb * kBlk + 2 * cblk);
        for (int b = 0; b < nrb; ++b) tma_load_2d(sDv + b * kBlk, &tmDv, 64 * b, h * DH, &B.fin_b);
        for (int b = 0; b < 2; ++b) tma_load_2d(sCv + b * cblk, &tmCv, h * DH + 64 * b, 0, &B.fin_b);
        mbar_wait(&B.fin_b, 0, nullptr, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ), aDk = smem_u32(sDk), aCk = smem_u32(sCk);
      const uint32_t aQt = smem_u32(sQt), aK = smem_u32(sKc), aV = smem_u32(sVc), aOH = smem_u32(sOH);
      bool ok = mbar_wait(&B.pro_full, 0, abort, err);
      if (ok) {
        tc_fence_after();
        // Q~ = Q D_{K,h} (B: N = r contiguous -> MN-major); QC = Q C_{K,h}^T (B K-major)
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          const uint32_t offA = (ks >> 2) * kBlk + (ks & 3) * 32;
          mma_ss(tbase + TM_OT, sdesc_sw128(aQ + offA, 16, 1024), sdesc_sw128(aDk + ks * 2048, kBlk, 1024),
                 idesc_bf16(128, r, false, true), ks > 0);
          mma_ss(tbase + TM_OT + r, sdesc_sw128(aQ + offA, 16, 1024),
                 sdesc_sw128(aCk + (ks >> 2) * cblk + (ks & 3) * 32, 16, 1024), idesc_bf16(128, C, false, false),
                 ks > 0);
        }
        mma_commit(&B.pro_done);
        ok = mbar_wait(&B.qt_ready, 0, abort, err);
      }
      // Two MMA streams polled with non-blocking tests and issued as soon as
      // their inputs are ready, so that neither waits behind the other:
      // scores S'_j = Q~ codes_K^T (S buffer j & 1, which last held P of
      // tile j - 2) and values O~ += (P s_V) codes_V, P_C += P onehot.
      int js = 0, jv = 0;
      uint64_t t_last = globaltimer();
      while (ok && jv < ntiles) {
        bool progress = false;
        // ---- values stream (frees the V code buffer for the unpackers)
        if (jv < js && mbar_test(&B.p_full[jv & 1], (jv >> 1) & 1) && mbar_test(&B.vc_full, jv & 1)) {
          LOW_TRACE(1, jv);
          tc_fence_after();
          const uint32_t sb = tbase + TM_S0 + (jv & 1) * 128;
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint32_t pc = sb + 32 * (ks >> 1) + 8 * (ks & 1);
            const uint32_t acc = (jv > 0 || ks > 0);
            mma_ts(tbase + TM_OT, pc + 16, sdesc_sw128(aV + ks * 2048, kBlk, 1024), idesc_bf16(128, r, false, true),
                   acc);
            mma_ts(tbase + TM_OT + r, pc, sdesc_sw128(aOH + ks * 2048, kBlk, 1024), idesc_bf16(128, C, false, true),
                   acc);
          }
          mma_commit(&B.pv_done[jv & 1]);
          mma_commit(&B.v_empty);
          ++jv;
          progress = true;
        }
        // ---- scores stream
        if (js < ntiles && mbar_test(&B.kc_full, js & 1) &&
            (js < 2 || mbar_test(&B.pv_done[js & 1], ((js - 2) >> 1) & 1))) {
          LOW_TRACE(0, js);
          tc_fence_after();
          const uint32_t dS = tbase + TM_S0 + (js & 1) * 128;
          for (int ks = 0; ks < r / 16; ++ks) {
            const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
            mma_ss(dS, sdesc_sw128(aQt + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024),
                   idesc_bf16(128, 128, false, false), ks > 0);
          }
          mma_commit(&B.s_full[js & 1]);
          mma_commit(&B.kc_empty);
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
      if (ok) mma_commit(&B.last_done);
      // restore: O = [O~/l | P_C/l] [D_{V,h} | C_{V,h}^T]^T
      if (ok && mbar_wait(&B.fin_a, 0, abort, err) && mbar_wait(&B.fin_b, 0, abort, err)) {
        tc_fence_after();
        const uint32_t aAo = smem_u32(sAo), aAp = smem_u32(sAp), aDv = smem_u32(sDv), aCv = smem_u32(sCv);
        for (int ks = 0; ks < r / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBlk + (ks & 3) * 32;
          mma_ss(tbase + TM_S0, sdesc_sw128(aAo + off, 16, 1024), sdesc_sw128(aDv + off, 16, 1024),
                 idesc_bf16(128, 128, false, false), ks > 0);
        }
        for (int ks = 0; ks < C / 16; ++ks) {
          mma_ss(tbase + TM_S0, sdesc_sw128(aAp + (ks & 3) * 32, 16, 1024),
                 sdesc_sw128(aCv + ks * 2048, cblk, 1024), idesc_bf16(128, 128, false, true), 1);
        }
        mma_commit(&B.fin_done);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------- key-side unpack: two keys per thread ----------------
    // Keys t and t + 64 of every tile: their K codes into the K buffer (freed
    // by the previous tile's scores MMA) and their center id and scales into
    // the per-key arrays of the tile's parity, which the softmax of tile
    // j - 2 read last.  The value side runs in warps 4..7 on its own chain,
    // so the next tile's scores never wait behind this tile's value MMAs.
    // Each key's ids, scales and codes of tile j + 1 are loaded into
    // registers while tile j is unpacked.
    const int t = (warp - 2) * 32 + lane;
    const int cw = r / 32;  // uint4 words of packed codes per key
    struct KeyK {
      int ak;
      float sk, sv;
      uint4 ck[kMaxCodeWords];
    };
    auto load_key = [&](int j, int key, KeyK &d) {
      const int64_t tt = A.t0 + (int64_t)j * BN + key;
      const bool valid = (int64_t)j * BN + key < A.T;
      const int ak = valid ? (int)A.idk[tt] : 0;
      d.ak = ak < C ? ak : C - 1;
      d.sk = valid ? __half2float(A.sk[tt]) : 0.f;
      d.sv = valid ? __half2float(A.sv[tt]) : 0.f;
      const uint4 *pk = reinterpret_cast<const uint4 *>(A.codk + tt * (r / 2));
#pragma unroll
      for (int q = 0; q < kMaxCodeWords; ++q) d.ck[q] = (q < cw && valid) ? __ldg(pk + q) : make_uint4(0, 0, 0, 0);
    };
    auto store_key = [&](int j, int key, const KeyK &d) {
#pragma unroll
      for (int q = 0; q < kMaxCodeWords; ++q) {
        if (q >= cw) break;
        const uint32_t w[4] = {d.ck[q].x, d.ck[q].y, d.ck[q].z, d.ck[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(sKc + sw128_offset(key, 32 * q + 8 * i, 128)) = unpack8(w[i]);
      }
      kAK[(j & 1) * 128 + key] = d.ak;
      kSK[(j & 1) * 128 + key] = d.sk;
      kSV[(j & 1) * 128 + key] = d.sv;
    };
    KeyK cur[2], nxt[2];
    bool ok = mbar_wait(&B.pro_done, 0, abort, err);  // prologue buffers alias the tiles
    if (ok && ntiles > 0) {
      load_key(0, t, cur[0]);
      load_key(0, t + 64, cur[1]);
    }
    for (int j = 0; ok && j < ntiles; ++j) {
      if (j + 1 < ntiles) {
        load_key(j + 1, t, nxt[0]);
        load_key(j + 1, t + 64, nxt[1]);
      }
      // the K buffer: tile j - 1's scores are done; the key arrays of this
      // parity: the softmax of tile j - 2 is done with them
      if (j >= 1 && !mbar_wait(&B.kc_empty, (j - 1) & 1, abort, err)) { ok = false; break; }
      if (j >= 2 && !mbar_wait(&B.p_full[j & 1], ((j - 2) >> 1) & 1, abort, err)) { ok = false; break; }
      if (t == 0) LOW_TRACE(4, j);
      store_key(j, t, cur[0]);
      store_key(j, t + 64, cur[1]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&B.kc_full);
        mbar_arrive(&B.info_full[j & 1]);
      }
      if (t == 0) LOW_TRACE(5, j);
      cur[0] = nxt[0];
      cur[1] = nxt[1];
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- value-side unpack (thread = key) ----------------
    // V codes and the one-hot of the value center into their buffers, freed
    // by the previous tile's value MMAs; tile j + 1's codes and id are loaded
    // into registers while tile j is unpacked.
    const int t = (warp - 4) * 32 + lane;
    const int cw = r / 32;
    struct KeyV {
      int av;
      uint4 cv[kMaxCodeWords];
    };
    auto load_key = [&](int j, KeyV &d) {
      const int64_t tt = A.t0 + (int64_t)j * BN + t;
      const bool valid = (int64_t)j * BN + t < A.T;
      const int av = valid ? (int)A.idv[tt] : 0;
      d.av = valid ? (av < C ? av : C - 1) : -1;  // -1: no one-hot entry
      const uint4 *pv = reinterpret_cast<const uint4 *>(A.codv + tt * (r / 2));
#pragma unroll
      for (int q = 0; q < kMaxCodeWords; ++q) d.cv[q] = (q < cw && valid) ? __ldg(pv + q) : make_uint4(0, 0, 0, 0);
    };
    KeyV cur, nxt;
    bool ok = mbar_wait(&B.pro_done, 0, abort, err);
    if (ok && ntiles > 0) load_key(0, cur);
    for (int j = 0; ok && j < ntiles; ++j) {
      if (j + 1 < ntiles) load_key(j + 1, nxt);
      if (j >= 1 && !mbar_wait(&B.v_empty, (j - 1) & 1, abort, err)) { ok = false; break; }
      if (t == 0) LOW_TRACE(6, j);
#pragma unroll
      for (int q = 0; q < kMaxCodeWords; ++q) {
        if (q >= cw) break;
        const uint32_t w[4] = {cur.cv[q].x, cur.cv[q].y, cur.cv[q].z, cur.cv[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(sVc + sw128_offset(t, 32 * q + 8 * i, 128)) = unpack8(w[i]);
      }
      const int av = cur.av;
      for (int g = 0; g < C / 8; ++g) {
        uint4 z = make_uint4(0, 0, 0, 0);
        if (av >= 0 && (av >> 3) == g) {
          const uint32_t one = 0x3F80u << (16 * (av & 1));  // bf16 1.0 in the right half
          const int wsel = (av & 7) >> 1;
          if (wsel == 0) z.x = one;
          else if (wsel == 1) z.y = one;
          else if (wsel == 2) z.z = one;
          else z.w = one;
        }
        *reinterpret_cast<uint4 *>(sOH + sw128_offset(t, 8 * g, 128)) = z;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.vc_full);
      if (t == 0) LOW_TRACE(7, j);
      cur = nxt;
    }
  } else if (warp >= 8) {
    // ---------------- softmax (thread = query row) ----------------
    const int row = (warp - 8) * 32 + lane;
    const float zs = A.zscale;
    bool ok = mbar_wait(&B.pro_done, 0, abort, err);
    if (ok) {
      tc_fence_after();
      uint32_t v[32];
      // Q~ * tau*log2e -> bf16, stored in the unpack order of the codes
      for (int c0 = 0; c0 < r; c0 += 32) {
        tmem_ld32(tmem_lane_addr(tbase, warp, TM_OT + c0), v);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float *f = reinterpret_cast<const float *>(v + 8 * g);
          const uint4 o = make_uint4(pack_bf16x2(f[0] * zs, f[4] * zs), pack_bf16x2(f[1] * zs, f[5] * zs),
                                     pack_bf16x2(f[2] * zs, f[6] * zs), pack_bf16x2(f[3] * zs, f[7] * zs));
          *reinterpret_cast<uint4 *>(sQt + sw128_offset(row, c0 + 8 * g, 128)) = o;
        }
      }
      for (int c0 = 0; c0 < C; c0 += 16) {
        uint32_t u[16];
        tmem_ld16(tmem_lane_addr(tbase, warp, TM_OT + r + c0), u);
#pragma unroll
        for (int i = 0; i < 16; ++i) sQC[row * (C + 1) + c0 + i] = __uint_as_float(u[i]) * zs;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.qt_ready);
    }
    const float *qc = sQC + row * (C + 1);
    RowState st{-INFINITY, 0.f};
    for (int j = 0; ok && j < ntiles; ++j) {
      if (!mbar_wait(&B.s_full[j & 1], (j >> 1) & 1, abort, err)) { ok = false; break; }
      if (!mbar_wait(&B.info_full[j & 1], (j >> 1) & 1, abort, err)) { ok = false; break; }
      if (row == 0) LOW_TRACE(2, j);
      tc_fence_after();
      const uint32_t sb = TM_S0 + (j & 1) * 128;
      const int *aKj = kAK + (j & 1) * 128;
      const float *sKj = kSK + (j & 1) * 128, *sVj = kSV + (j & 1) * 128;
      const int64_t rem = A.T - (int64_t)j * BN;
      const int nk = rem < BN ? (int)rem : BN;
      const bool full = nk >= BN;
      uint32_t v[32];
      // pass 1: z = s_K S' + QC[a_K] per key (one gather per key), row max;
      // z replaces S' in TMEM for pass 2
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const uint32_t taddr = tmem_lane_addr(tbase, warp, sb + 32 * c);
        tmem_ld32(taddr, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int4 a4 = *reinterpret_cast<const int4 *>(aKj + 32 * c + 4 * q);
          const float4 s4 = *reinterpret_cast<const float4 *>(sKj + 32 * c + 4 * q);
          const int aa[4] = {a4.x, a4.y, a4.z, a4.w};
          const float ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = 4 * q + u;
            const float z = fmaf(__uint_as_float(v[i]), ss[u], qc[aa[u]]);
            v[i] = __float_as_uint(z);
            if (full) mx4[u] = fmaxf(mx4[u], z);
            else mx4[u] = (32 * c + i < nk) ? fmaxf(mx4[u], z) : mx4[u];
          }
        }
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) { lo[i] = v[i]; hi[i] = v[16 + i]; }
        tmem_st16(taddr, lo);
        tmem_st16(taddr + 16, hi);
      }
      tmem_st_wait();
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      float corr = 1.f;
      const bool need = mx > st.m + kRescaleLog2;
      if (need) {
        corr = (st.m == -INFINITY) ? 0.f : ex2(st.m - mx);
        st.l *= corr;
        st.m = mx;
      }
      const bool wr = __any_sync(0xffffffffu, need) != 0;
      if (row == 0) LOW_TRACE(8, j);
      const float m = st.m;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      // pass 2: P and P * s_V, interleaved per 32 keys over the z columns
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tmem_lane_addr(tbase, warp, sb + 32 * c), v);
        uint32_t pp[16], ps[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 sv4 = *reinterpret_cast<const float4 *>(sVj + 32 * c + 4 * q);
          const float svv[4] = {sv4.x, sv4.y, sv4.z, sv4.w};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int i = 2 * q + h2;  // pair index within the chunk
            const int k0 = 32 * c + 2 * i;
            float p0 = ex2(__uint_as_float(v[2 * i]) - m);
            float p1 = ex2(__uint_as_float(v[2 * i + 1]) - m);
            if (!full) {
              p0 = (k0 < nk) ? p0 : 0.f;
              p1 = (k0 + 1 < nk) ? p1 : 0.f;
            }
            ls[i & 3] += p0 + p1;
            pp[i] = pack_bf16x2(p0, p1);
            ps[i] = pack_bf16x2(p0 * svv[2 * h2], p1 * svv[2 * h2 + 1]);
          }
        }
        tmem_st16(tmem_lane_addr(tbase, warp, sb + 32 * c), pp);
        tmem_st16(tmem_lane_addr(tbase, warp, sb + 32 * c + 16), ps);
      }
      const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_st_wait();
      st.l += lsum;
      if (j > 0 && wr) {
        if (!mbar_wait(&B.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort, err)) { ok = false; break; }
        tc_fence_after();
        rescale_cols(tbase, warp, TM_OT, r + C, corr);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_full[j & 1]);
      if (row == 0) LOW_TRACE(3, j);
    }
    // restore operands: [O~ | P_C] / l in bf16 (O~ un-permuted)
    if (ok && mbar_wait(&B.last_done, 0, abort, err)) {
      tc_fence_after();
      const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
      uint32_t v[32];
      for (int c0 = 0; c0 < r; c0 += 32) {
        tmem_ld32(tmem_lane_addr(tbase, warp, TM_OT + c0), v);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          // stored position p holds code (0,4,1,5,2,6,3,7)[p]
          const float *f = reinterpret_cast<const float *>(v + 8 * g);
          const uint4 o = make_uint4(pack_bf16x2(f[0] * inv, f[2] * inv), pack_bf16x2(f[4] * inv, f[6] * inv),
                                     pack_bf16x2(f[1] * inv, f[3] * inv), pack_bf16x2(f[5] * inv, f[7] * inv));
          *reinterpret_cast<uint4 *>(sAo + sw128_offset(row, c0 + 8 * g, 128)) = o;
        }
      }
      for (int c0 = 0; c0 < C; c0 += 16) {
        uint32_t u[16];
        tmem_ld16(tmem_lane_addr(tbase, warp, TM_OT + r + c0), u);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const float *f = reinterpret_cast<const float *>(u + 8 * g);
          const uint4 o = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                                     pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
          *reinterpret_cast<uint4 *>(sAp + sw128_offset(row, c0 + 8 * g, 128)) = o;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.fin_a);
      if (mbar_wait(&B.fin_done, 0, abort, err)) {
        tc_fence_after();
        const int64_t qrow = q0 + row;
        float *dst = A.O + (qrow * A.H + h) * DH;
        for (int c0 = 0; c0 < DH; c0 += 32) {
          tmem_ld32(tmem_lane_addr(tbase, warp, TM_S0 + c0), v);
          if (qrow < A.Tq) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4 *>(dst + c0 + i) =
                  make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                              __uint_as_float(v[i + 3]));
          }
        }
        if (qrow < A.Tq) A.L[(int64_t)h * A.Tq + qrow] = st.l > 0.f ? (st.m + log2f(st.l)) * kLn2 : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
}

}  // namespace

#ifdef NANOKV_TRACE
extern "C" int nanokv_debug_low_trace(void *host, size_t bytes) {
  if (bytes < sizeof(g_low_trace)) return -1;
  return cudaMemcpyFromSymbol(host, g_low_trace, sizeof(g_low_trace)) == cudaSuccess ? 0 : -3;
}
#endif

bool tc_low_supported(const Codec &ck, const Codec &cv) {
  return ck.prec == PREC_BF16 && ck.d == DH && ck.r == cv.r && ck.C == cv.C && ck.r % 64 == 0 &&
         ck.r <= 192 && ck.C % 16 == 0 && ck.C <= 64;
}

static size_t low_smem(int r, int C) {
  const int nrb = r / 64;
  return (size_t)(3 * nrb + 1) * kBlk + (size_t)128 * (C + 1) * 4 + 3 * 2 * 128 * 4 + 1024;
}

cudaError_t tc_attend_low(const void *q, int64_t Tq, const Codec &ck, const Codec &cv, const Hist &hk,
                          const Hist &hv, int64_t t0, int64_t T, float tau, Part out, cudaStream_t st,
                          HeadSel hs) {
  if (Tq == 0 || T == 0) return cudaSuccess;
  const int J = ck.H * DH;
  CUtensorMap mq, mdk, mck, mdv, mcv;
  if (!make_tmap_bf16_2d(&mq, q, Tq, J, J, 128) || !make_tmap_bf16_2d(&mdk, ck.D, J, ck.r, ck.r, 128) ||
      !make_tmap_bf16_2d(&mck, ck.centers, ck.C, J, J, ck.C) ||
      !make_tmap_bf16_2d(&mdv, cv.D, J, cv.r, cv.r, 128) ||
      !make_tmap_bf16_2d(&mcv, cv.centers, cv.C, J, J, cv.C))
    return cudaErrorInvalidValue;
  LowArgs a;
  a.Dk = (const __nv_bfloat16 *)ck.D;
  a.Dv = (const __nv_bfloat16 *)cv.D;
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
  a.C = ck.C;
  a.zscale = tau * kLog2e;
  a.O = out.O;
  a.L = out.LSE;
  a.err = error_word_ptr();
  a.head_map = hs.map;
  const size_t smem = low_smem(ck.r, ck.C);
  ensure_smem((const void *)tc_low_kernel, (int)smem);
  dim3 grid((unsigned)((Tq + BM - 1) / BM), (unsigned)(hs.map ? hs.n : ck.H));
  tc_low_kernel<<<grid, 384, smem, st>>>(mq, mdk, mck, mdv, mcv, a);
  return cudaGetLastError();
}

}  // namespace nanokv
