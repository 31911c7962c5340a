// Tensor-core attention of the query chunk over the current, uncompressed
// chunk (the third branch merged by LSE; NanoKV Fig. 4(d)).  One CTA per
// (128-row query tile, head):
//   warp 0      TMA producer: Q once, then K tiles (3 stages)
//   warp 1      MMA issuer:   S = Q K^T (SS), O += P V (P read from TMEM)
//   warp 2      TMA producer: V tiles (2 stages)
//   warps 4..11 softmax:      two threads per query row (TMEM lane), each
//                             owning 64 of the tile's 128 keys
// S and O accumulate in TMEM; P overwrites S as bf16.  A K stage is released
// by the score MMAs that read it and a V stage by the value MMAs, and the two
// streams have their own producers, so the next tiles' keys load while the
// softmax runs instead of after the previous value MMA.  Every wait is
// bounded.
#include "tc_common.cuh"

namespace nanokv {

using namespace sm100;
using namespace tc;

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                       uint64_t row_stride_elems, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                     uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
                   es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

constexpr int DH = 128;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one [128 x 128] bf16 operand tile
constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);
constexpr uint32_t TM_O = 0, TM_S = 128, TM_COLS = 512;  // S: two 128-column buffers
constexpr int KST = 3;                                     // K stages (V has 2)

struct DenseBars {
  uint64_t q_full, k_full[KST], k_empty[KST], v_full[2], v_empty[2], s_full[2], p_full[2], pv_done;
  uint32_t tmem_base;
  int abort;
  uint64_t xbar[2], lbar;  // row-max exchange per tile parity; final row-sum exchange
  float xmax[2][2][128];   // [tile parity][half][row] partial row maxima
  float lsum[2][128];      // [half][row] final partial row sums
};

__global__ void __launch_bounds__(384, 1)
    tc_dense_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, int64_t Tq, int64_t T, int H,
                    float zscale, float *__restrict__ Oout, float *__restrict__ Lout,
                    unsigned *err) {
  extern __shared__ uint8_t smraw[];
  uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = sm;
  uint8_t *sK[KST] = {sm + kTileBytes, sm + 2 * kTileBytes, sm + 3 * kTileBytes};
  uint8_t *sV[2] = {sm + 4 * kTileBytes, sm + 5 * kTileBytes};
  __shared__ DenseBars B;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t q0 = (int64_t)blockIdx.x * BM;
  const int ntiles = (int)((T + BN - 1) / BN);
  volatile int *abort = &B.abort;

  if (threadIdx.x == 0) {
    mbar_init(&B.q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&B.k_full[s], 1);
      mbar_init(&B.k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.v_full[s], 1);
      mbar_init(&B.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.s_full[s], 1);
      mbar_init(&B.p_full[s], 8);
      mbar_init(&B.xbar[s], 8);
    }
    mbar_init(&B.pv_done, 1);
    mbar_init(&B.lbar, 8);
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
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&B.q_full, kTileBytes);
      tma_load_2d(sQ, &tmQ, h * DH, (int)q0, &B.q_full);
      tma_load_2d(sQ + kTileBytes / 2, &tmQ, h * DH + 64, (int)q0, &B.q_full);
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % KST;
        if (j >= KST && !mbar_wait(&B.k_empty[s], ((j / KST) - 1) & 1, abort, err)) break;
        const int k0 = j * BN;
        mbar_arrive_expect_tx(&B.k_full[s], kTileBytes);
        tma_load_2d(sK[s], &tmK, h * DH, k0, &B.k_full[s]);
        tma_load_2d(sK[s] + kTileBytes / 2, &tmK, h * DH + 64, k0, &B.k_full[s]);
        issued = j + 1;
      }
      // drain: every issued copy completes before the CTA may exit
      mbar_wait(&B.q_full, 0, nullptr, nullptr);
      for (int j = (issued > KST ? issued - KST : 0); j < issued; ++j)
        mbar_wait(&B.k_full[j % KST], (j / KST) & 1, nullptr, nullptr);
    }
  } else if (warp == 2) {
    // ---------------- TMA producer: values ----------------
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&B.v_empty[s], ((j >> 1) - 1) & 1, abort, err)) break;
        const int k0 = j * BN;
        mbar_arrive_expect_tx(&B.v_full[s], kTileBytes);
        tma_load_2d(sV[s], &tmV, h * DH, k0, &B.v_full[s]);
        tma_load_2d(sV[s] + kTileBytes / 2, &tmV, h * DH + 64, k0, &B.v_full[s]);
        issued = j + 1;
      }
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
        mbar_wait(&B.v_full[j & 1], (j >> 1) & 1, nullptr, nullptr);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool ok = mbar_wait(&B.q_full, 0, abort, err);
      const uint32_t aQ = smem_u32(sQ);
      auto scores = [&](int j) -> bool {
        const int s = j & 1, ks3 = j % KST;
        if (!mbar_wait(&B.k_full[ks3], (j / KST) & 1, abort, err)) return false;
        // the S buffer of tile j last held P of tile j - 2
        if (j >= 2 && !mbar_wait(&B.pv_done, (j - 2) & 1, abort, err)) return false;
        tc_fence_after();
        const uint32_t aK = smem_u32(sK[ks3]);
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          const uint32_t off = (ks >> 2) * (kTileBytes / 2) + (ks & 3) * 32;
          mma_ss(tbase + TM_S + s * 128, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024),
                 IDESC_S, ks > 0);
        }
        mma_commit(&B.s_full[s]);
        mma_commit(&B.k_empty[ks3]);
        return true;
      };
      auto values = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(&B.p_full[s], (j >> 1) & 1, abort, err)) return false;
        if (!mbar_wait(&B.v_full[s], (j >> 1) & 1, abort, err)) return false;
        tc_fence_after();
        const uint32_t aV = smem_u32(sV[s]);
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_ts(tbase + TM_O, tbase + TM_S + s * 128 + ks * 8,
                 sdesc_sw128(aV + ks * 2048, kTileBytes / 2, 1024), IDESC_PV, (j > 0 || ks > 0));
        mma_commit(&B.pv_done);
        mma_commit(&B.v_empty[s]);
        return true;
      };
      if (ok) ok = scores(0);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles && !scores(j + 1)) break;
        if (!values(j)) break;
      }
    }
  } else if (warp >= 4) {
    // ---------------- softmax (two threads per query row) ----------------
    const int half = (warp - 4) >> 2;  // 0: keys 0..63 of a tile, 1: keys 64..127
    const int row = (warp & 3) * 32 + lane;
    RowState st{-INFINITY, 0.f};
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!mbar_wait(&B.s_full[j & 1], (j >> 1) & 1, abort, err)) { ok = false; break; }
      tc_fence_after();
      const int64_t rem = T - (int64_t)j * BN;
      const int nk = rem < BN ? (int)rem : BN;
      bool wr;
      float corr;
      if (!softmax_tile_half(tbase, warp, TM_S + (j & 1) * 128, nk, half, row, &B.xmax[j & 1][0][0],
                             &B.xbar[j & 1], (j >> 1) & 1, abort, err, zscale, st, wr, corr)) {
        ok = false;
        break;
      }
      if (j > 0 && wr) {
        if (!mbar_wait(&B.pv_done, (j - 1) & 1, abort, err)) { ok = false; break; }
        tc_fence_after();
        rescale_cols(tbase, warp, TM_O + 64 * half, 64, corr);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_full[j & 1]);
    }
    // the value MMAs may trail the softmax by two tiles: wait for the last two
    // phases in order so that a parity can never be mistaken for an older one
    if (ok && ntiles >= 2) ok = mbar_wait(&B.pv_done, (ntiles - 2) & 1, abort, err);
    if (ok) ok = mbar_wait(&B.pv_done, (ntiles - 1) & 1, abort, err);
    B.lsum[half][row] = st.l;
    __syncwarp();
    if (lane == 0) mbar_arrive(&B.lbar);
    if (ok) ok = mbar_wait(&B.lbar, 0, abort, err);
    if (ok) {
      tc_fence_after();
      const float l = B.lsum[0][row] + B.lsum[1][row];
      const int64_t qrow = q0 + row;
      write_row_half(tbase, warp, TM_O, 64 * half, l > 0.f ? 1.f / l : 0.f, qrow, Tq, h, H, Oout);
      if (half == 0 && qrow < Tq) Lout[(int64_t)h * Tq + qrow] = l > 0.f ? (st.m + log2f(l)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
  pdl_wait_prior();
}

}  // namespace

bool tc_dense_supported(int prec, int d) { return prec == PREC_BF16 && d == DH; }

cudaError_t tc_attend_dense(const void *q, int64_t Tq, int H, int d, const void *k, const void *v,
                            int64_t T, float tau, Part out, cudaStream_t st, bool pdl) {
  if (Tq == 0 || T == 0) return cudaSuccess;
  const int J = H * d;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_bf16_2d(&mq, q, Tq, J, J, 128) || !make_tmap_bf16_2d(&mk, k, T, J, J, 128) ||
      !make_tmap_bf16_2d(&mv, v, T, J, J, 128))
    return cudaErrorInvalidValue;
  const size_t smem = (1 + KST + 2) * kTileBytes + 1024;
  ensure_smem((const void *)tc_dense_kernel, (int)smem);
  dim3 grid((unsigned)((Tq + BM - 1) / BM), (unsigned)H);
  return launch_k(tc_dense_kernel, grid, dim3(384), smem, st, pdl, mq, mk, mv, Tq, T, H, tau * kLog2e,
                  out.O, out.LSE, error_word_ptr());
}

}  // namespace nanokv
