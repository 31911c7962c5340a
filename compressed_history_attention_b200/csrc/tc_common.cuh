// Host helpers for the tensor-core kernels (tensor maps) and the per-row
// online-softmax / output stages shared by the attention kernels.
#pragma once

#include <cudaTypedefs.h>

#include "sm100.cuh"
#include "tc.cuh"

namespace nanokv {

// ---------------------------------------------------------------------------
// host: 2-D bf16 tensor map (row-major [rows, cols], row stride in elements),
// box [64 cols x box_rows], 128-byte swizzle, zero fill out of bounds.
// ---------------------------------------------------------------------------
bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                       uint64_t row_stride_elems, uint32_t box_rows);
bool make_tmap_u8_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                     uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows);

// Launches `kern` on `st`; with `pdl` the launch may overlap the tail of the
// previous kernel in the stream (programmatic dependent launch).  Kernels
// launched this way never read the previous kernel's output and wait for it
// (griddepcontrol.wait) before they exit, so stream order still holds for
// whatever comes after them.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

namespace tc {

constexpr int BM = 128;  // query rows per CTA (TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
// lazy rescaling: keep the running max until a row's max grows by more than
// this many powers of two (probabilities then stay below 2^kRescaleLog2)
constexpr float kRescaleLog2 = 8.0f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// 8 packed INT4 codes (one 32-bit word, code i in bits [4i, 4i+4)) -> 8 bf16
// in the order (n0,n4), (n1,n5), (n2,n6), (n3,n7): position p of the group
// holds code (0,4,1,5,2,6,3,7)[p].  (n XOR 8) | 0x4300 is the bf16 bit
// pattern of 128 + (n + 8) for a two's-complement nibble n; subtracting 136
// leaves n exactly.
__device__ __forceinline__ uint4 unpack8(uint32_t w) {
  const __nv_bfloat162 bias = __floats2bfloat162_rn(136.f, 136.f);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t b = ((w >> (4 * i)) & 0x000F000Fu) ^ 0x43084308u;
    __nv_bfloat162 v = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&b), bias);
    o[i] = *reinterpret_cast<uint32_t *>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// TMEM address of (lane base of this warp's quarter, column)
__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base, int warp, uint32_t col) {
  return base + ((uint32_t)((warp & 3) * 32) << 16) + col;
}

// Online-softmax state of one query row (one thread), log2 domain.
struct RowState {
  float m;  // running max of the scaled scores (log2 units)
  float l;  // running sum of 2^(z - m)
};

#ifdef NANOKV_TRACE
// debug builds only: clock64 stamps of the softmax stages of one row
__device__ unsigned long long g_softmax_trace[8][128];
#define SOFTMAX_TRACE(i, tj)                                            \
  do {                                                                  \
    if ((tj) >= 0 && (tj) < 128) g_softmax_trace[i][tj] = clock64();    \
  } while (0)
#else
#define SOFTMAX_TRACE(i, tj) \
  do {                       \
  } while (0)
#endif

// One key tile of the online softmax for the calling thread's row.
// Reads S (fp32, 128 columns at s_col), writes P as packed bf16 into the first
// 64 of those columns, updates the row state.  `nk` valid keys; `zscale`
// multiplies raw scores into log2 units.  Returns the factor by which the
// caller must rescale O (1 if none); *rescale tells whether any row of the
// warp needs it.  Full tiles take a compact loop over 32-column chunks (the
// kernels that call this run many warp roles at once, and their unrolled
// code competes for the instruction cache); a partial last tile takes a
// rolled, masked path.
static __device__ __noinline__ float softmax_tile_partial(uint32_t tbase, int warp, uint32_t s_col, int nk, float zscale,
                                                   RowState &st, bool &warp_rescale) {
  float mx = -INFINITY;
  uint32_t r32[32];
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    sm100::tmem_ld32(tmem_lane_addr(tbase, warp, s_col + 32 * c), r32);
#pragma unroll
    for (int i = 0; i < 32; ++i) mx = (32 * c + i < nk) ? fmaxf(mx, __uint_as_float(r32[i])) : mx;
  }
  mx *= zscale;
  float corr = 1.f;
  const bool need = mx > st.m + kRescaleLog2;
  if (need) {
    corr = (st.m == -INFINITY) ? 0.f : ex2(st.m - mx);
    st.l *= corr;
    st.m = mx;
  }
  warp_rescale = __any_sync(0xffffffffu, need) != 0;
  const float m = st.m;
  float ls = 0.f;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    sm100::tmem_ld32(tmem_lane_addr(tbase, warp, s_col + 32 * c), r32);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int k0 = 32 * c + 2 * i;
      const float p0 = (k0 < nk) ? ex2(fmaf(__uint_as_float(r32[2 * i]), zscale, -m)) : 0.f;
      const float p1 = (k0 + 1 < nk) ? ex2(fmaf(__uint_as_float(r32[2 * i + 1]), zscale, -m)) : 0.f;
      ls += p0 + p1;
      pk[i] = pack_bf16x2(p0, p1);
    }
    sm100::tmem_st16(tmem_lane_addr(tbase, warp, s_col + 16 * c), pk);
  }
  sm100::tmem_st_wait();
  st.l += ls;
  return corr;
}

__device__ __forceinline__ float softmax_tile(uint32_t tbase, int warp, uint32_t s_col, int nk,
                                              float zscale, RowState &st, bool &warp_rescale,
                                              int trace_j = -1) {
  if (nk < 128) return softmax_tile_partial(tbase, warp, s_col, nk, zscale, st, warp_rescale);
  // pass 1: row max over the tile, four independent chains
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  SOFTMAX_TRACE(0, trace_j);
  uint32_t r32[32];
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    sm100::tmem_ld32(tmem_lane_addr(tbase, warp, s_col + 32 * c), r32);
#pragma unroll
    for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(r32[i]));
  }
  // scores are scaled after the max (zscale > 0 keeps the order)
  const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * zscale;
  float corr = 1.f;
  const bool need = mx > st.m + kRescaleLog2;  // also true when st.m == -inf
  if (need) {
    corr = (st.m == -INFINITY) ? 0.f : ex2(st.m - mx);
    st.l *= corr;
    st.m = mx;
  }
  warp_rescale = __any_sync(0xffffffffu, need) != 0;
  SOFTMAX_TRACE(1, trace_j);
  const float m = st.m;
  float ls[4] = {0.f, 0.f, 0.f, 0.f};
  // pass 2 in 32-column chunks
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    sm100::tmem_ld32(tmem_lane_addr(tbase, warp, s_col + 32 * c), r32);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float p0 = ex2(fmaf(__uint_as_float(r32[2 * i]), zscale, -m));
      const float p1 = ex2(fmaf(__uint_as_float(r32[2 * i + 1]), zscale, -m));
      ls[i & 3] += p0 + p1;
      pk[i] = pack_bf16x2(p0, p1);
    }
    // P of S columns [32c, 32c + 32) goes to columns [16c, 16c + 16), all of
    // which were read by this chunk or an earlier one
    sm100::tmem_st16(tmem_lane_addr(tbase, warp, s_col + 16 * c), pk);
  }
  sm100::tmem_st_wait();
  SOFTMAX_TRACE(3, trace_j);
  st.l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
  return corr;
}

// Half-row variant of softmax_tile: two threads share a query row, thread
// `half` owning S columns [64 half, 64 half + 64).  The two partial maxima meet
// in `xmax` (shared, [2 halves][128 rows], one buffer per tile parity): every
// softmax warp arrives on `xbar` (count: all softmax warps) and waits for its
// phase `parity` with the usual bound.  The scores stay in registers between
// the passes.  P of this half goes to columns [32 half, 32 half + 32) of the S
// buffer (columns the other half had read before arriving).  st.l accumulates
// this half's share of the row sum.  Returns false if the exchange gave up.
__device__ __forceinline__ bool softmax_tile_half(uint32_t tbase, int warp, uint32_t s_col, int nk, int half,
                                                  int row, float *xmax, uint64_t *xbar, uint32_t parity,
                                                  volatile int *abort, unsigned *err, float zscale,
                                                  RowState &st, bool &warp_rescale, float &corr) {
  uint32_t r[64];
  sm100::tmem_ld64(tmem_lane_addr(tbase, warp, s_col + 64 * half), r);
  const int base = 64 * half;
  const bool full = nk >= 128;
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  if (full) {
#pragma unroll
    for (int i = 0; i < 64; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(r[i]));
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i) mx4[i & 3] = (base + i < nk) ? fmaxf(mx4[i & 3], __uint_as_float(r[i])) : mx4[i & 3];
  }
  xmax[half * 128 + row] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
  __syncwarp();
  if ((threadIdx.x & 31) == 0) sm100::mbar_arrive(xbar);
  if (!sm100::mbar_wait(xbar, parity, abort, err)) return false;
  const float mx = fmaxf(xmax[row], xmax[128 + row]) * zscale;
  corr = 1.f;
  const bool need = mx > st.m + kRescaleLog2;  // identical in both halves
  if (need) {
    corr = (st.m == -INFINITY) ? 0.f : ex2(st.m - mx);
    st.l *= corr;
    st.m = mx;
  }
  warp_rescale = __any_sync(0xffffffffu, need) != 0;
  const float m = st.m;
  float ls[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t pk[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int k0 = base + 2 * i;
    float p0 = ex2(fmaf(__uint_as_float(r[2 * i]), zscale, -m));
    float p1 = ex2(fmaf(__uint_as_float(r[2 * i + 1]), zscale, -m));
    if (!full) {
      p0 = (k0 < nk) ? p0 : 0.f;
      p1 = (k0 + 1 < nk) ? p1 : 0.f;
    }
    ls[i & 3] += p0 + p1;
    pk[i] = pack_bf16x2(p0, p1);
  }
  uint32_t lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) { lo[i] = pk[i]; hi[i] = pk[16 + i]; }
  sm100::tmem_st16(tmem_lane_addr(tbase, warp, s_col + 32 * half), lo);
  sm100::tmem_st16(tmem_lane_addr(tbase, warp, s_col + 32 * half + 16), hi);
  sm100::tmem_st_wait();
  st.l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
  return true;
}

// Multiplies `ncols` (multiple of 16) fp32 columns of this thread's row at col by f.
__device__ __forceinline__ void rescale_cols(uint32_t tbase, int warp, uint32_t col, int ncols, float f) {
  uint32_t v[16];
  for (int c = 0; c < ncols; c += 16) {
    const uint32_t a = tmem_lane_addr(tbase, warp, col + c);
    sm100::tmem_ld16(a, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
    sm100::tmem_st16(a, v);
  }
  sm100::tmem_st_wait();
}

// Writes columns [col0, col0 + 64) of the normalised O row (fp32 partials).
__device__ __forceinline__ void write_row_half(uint32_t tbase, int warp, uint32_t o_col, int col0, float inv,
                                               int64_t row, int64_t Tq, int h, int H, float *__restrict__ O) {
  uint32_t r[64];
  sm100::tmem_ld64(tmem_lane_addr(tbase, warp, o_col + col0), r);
  if (row < Tq) {
    float *dst = O + (row * H + h) * 128 + col0;
#pragma unroll
    for (int i = 0; i < 64; i += 4)
      *reinterpret_cast<float4 *>(dst + i) = make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                                                         __uint_as_float(r[i + 2]) * inv,
                                                         __uint_as_float(r[i + 3]) * inv);
  }
}

// Multiplies this thread's O row (16 * n16 fp32 columns at o_col) by f.
__device__ __forceinline__ void rescale_o(uint32_t tbase, int warp, uint32_t o_col, float f, int n16 = 8) {
  uint32_t r[16];
#pragma unroll 1
  for (int c = 0; c < n16; ++c) {
    const uint32_t a = tmem_lane_addr(tbase, warp, o_col + 16 * c);
    sm100::tmem_ld16(a, r);
    sm100::tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
    sm100::tmem_st16(a, r);
  }
  sm100::tmem_st_wait();
}

// Writes the normalised O row and its natural-log LSE (fp32 partials).
__device__ __forceinline__ void write_row(uint32_t tbase, int warp, uint32_t o_col,
                                          const RowState &st, int64_t row, int64_t Tq, int h, int H,
                                          float *__restrict__ O, float *__restrict__ L) {
  const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
  uint32_t r[32];
  float *dst = O + (row * H + h) * 128;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    sm100::tmem_ld32(tmem_lane_addr(tbase, warp, o_col + 32 * c), r);
    sm100::tmem_ld_wait();
    if (row < Tq) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 v = make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                               __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
        *reinterpret_cast<float4 *>(dst + 32 * c + i) = v;
      }
    }
  }
  if (row < Tq) L[(int64_t)h * Tq + row] = st.l > 0.f ? (st.m + log2f(st.l)) * kLn2 : -INFINITY;
}

// Reduced attention dimension: normalises this thread's o~ row (DHR fp32
// columns at o_col) and writes the restored row O = W_h o~ (128 columns,
// fp32 accumulation) and the LSE.  Wh: the head's value map [128, 128] bf16,
// row-major, columns [0, DHR) used; every lane reads the same map element at
// the same time.
template <int DHR>
__device__ __forceinline__ void write_row_restored(uint32_t tbase, int warp, uint32_t o_col, const RowState &st,
                                                   int64_t row, int64_t Tq, int h, int H,
                                                   const __nv_bfloat16 *__restrict__ Wh, float *__restrict__ O,
                                                   float *__restrict__ L) {
  const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
  float ot[DHR];
#pragma unroll
  for (int c = 0; c < DHR / 32; ++c) {
    uint32_t r[32];
    sm100::tmem_ld32(tmem_lane_addr(tbase, warp, o_col + 32 * c), r);
    sm100::tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) ot[32 * c + i] = __uint_as_float(r[i]) * inv;
  }
  float *dst = O + (row * H + h) * 128;
#pragma unroll 1
  for (int i = 0; i < 128; i += 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 *wrow = reinterpret_cast<const uint4 *>(Wh + (size_t)(i + u) * 128);
#pragma unroll
      for (int g = 0; g < DHR / 8; ++g) {
        const uint4 wv = __ldg(wrow + g);
        const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[k]));
          acc[u] = fmaf(f.x, ot[8 * g + 2 * k], acc[u]);
          acc[u] = fmaf(f.y, ot[8 * g + 2 * k + 1], acc[u]);
        }
      }
    }
    if (row < Tq) *reinterpret_cast<float4 *>(dst + i) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
  if (row < Tq) L[(int64_t)h * Tq + row] = st.l > 0.f ? (st.m + log2f(st.l)) * kLn2 : -INFINITY;
}

}  // namespace tc
}  // namespace nanokv
