// C ABI of libnanokv: argument validation, workspace layout, kernel selection.
#include "../../include/nanokv.h"
#include "common.cuh"
#include "sm100.cuh"

#include <nvtx3/nvToolsExt.h>
#include "tc.cuh"

#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

namespace nanokv {

// device error word (bounded waits that expired, bounds violations); read and
// cleared by nanokv_check
__device__ unsigned g_error_word = 0;

static thread_local std::string t_last_error;
static std::atomic<int> g_kernel_path{0};

static int fail(int status, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return status;
}

cudaError_t ensure_smem(const void *kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void *, int>, int>> done;  // ((kernel, device), bytes)
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (auto &e : done)
    if (e.first.first == kernel && e.first.second == dev) {
      if (e.second >= bytes) return cudaSuccess;
      const cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (r == cudaSuccess) e.second = bytes;
      return r;
    }
  const cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (r == cudaSuccess) done.push_back({{kernel, dev}, bytes});
  return r;
}

// records `msg` as the calling thread's last error and returns `status`
int set_error(int status, const char *msg) { return fail(status, "%s", msg); }

static int cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return NANOKV_OK;
  return fail(NANOKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------------------
// diagnostics: launch counts (always) and optional per-kernel event timing
// ---------------------------------------------------------------------------
static std::atomic<int> g_timing{0};
static std::atomic<int64_t> g_launches[NANOKV_K_COUNT];
struct TimingRec {
  int kid;
  cudaEvent_t a, b;
};
static std::mutex g_tmu;
static std::vector<TimingRec> g_recs;
static std::vector<cudaEvent_t> g_event_pool;

static cudaEvent_t event_get() {
  std::lock_guard<std::mutex> lk(g_tmu);
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// runs a launcher that issues `nk` kernels on `st`, counting and (optionally)
// timing them as kernel `kid`
template <class F>
static cudaError_t timed(int kid, int nk, cudaStream_t st, F &&launch) {
  g_launches[kid] += nk;
  if (!g_timing.load()) return launch();
  cudaEvent_t a = event_get(), b = event_get();
  cudaEventRecord(a, st);
  cudaError_t e = launch();
  cudaEventRecord(b, st);
  std::lock_guard<std::mutex> lk(g_tmu);
  g_recs.push_back({kid, a, b});
  return e;
}

// A wait that is never satisfied, bounded like every pipeline wait: thread 0
// initialises an mbarrier that nothing arrives on, polls it until `limit_ns`
// of wall time has passed, then records the timeout in the error word.
__global__ void selftest_wait_kernel(uint64_t limit_ns, unsigned *err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    const uint64_t t0 = sm100::globaltimer();
    bool done = false;
    while (!done) {
      done = sm100::mbar_test(&bar, 0);
      if (!done && sm100::globaltimer() - t0 > limit_ns) break;
    }
    if (!done) atomicOr(err, ERRW_TIMEOUT);
  }
}

// Helper streams on which the independent branch kernels of one attend call
// (low-dim, full-dim, current chunk) run concurrently.  The full-dim branch
// gets the highest priority, so its long two-CTA clusters are dispatched
// first; the current chunk gets the lowest, so its short CTAs fill the SMs
// the others leave idle (a partial last wave).  Created once per device and
// kept for the life of the process; callers on several host threads
// serialise on the mutex while they enqueue.
// Helper streams: 0 low-dim set, 1 full-dim set, 2 current chunk; 3 and 4
// the reduced-dimension heads of a routed call.
constexpr int kBranchStreams = 5;
struct BranchStreams {
  cudaStream_t s[kBranchStreams] = {};
  cudaEvent_t fork = nullptr, join[kBranchStreams] = {}, aux = nullptr;
  bool ready = false;
};
constexpr int kMaxDevices = 64;
static std::mutex g_bs_mu;
static BranchStreams g_bs[kMaxDevices];

// with g_bs_mu held
static cudaError_t branch_streams(BranchStreams **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  BranchStreams &b = g_bs[dev];
  if (!b.ready) {
    // creating streams and events is not a stream operation; let it proceed
    // if this thread is capturing a graph
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    cudaThreadExchangeStreamCaptureMode(&mode);
    int least = 0, greatest = 0;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    // numerically smaller is higher priority
    const int mid = greatest < least ? greatest + 1 : least;
    const int prio[kBranchStreams] = {mid, greatest, least, mid, mid};
    for (int i = 0; i < kBranchStreams && e == cudaSuccess; ++i)
      e = cudaStreamCreateWithPriority(&b.s[i], cudaStreamNonBlocking, prio[i]);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b.aux, cudaEventDisableTiming);
    for (int i = 0; i < kBranchStreams && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&b.join[i], cudaEventDisableTiming);
    cudaThreadExchangeStreamCaptureMode(&mode);
    if (e != cudaSuccess) return e;
    b.ready = true;
  }
  *out = &b;
  return cudaSuccess;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// One NVTX range per API call, so that a profiler timeline shows which
// library call launched which kernels (no effect without a profiler attached).
struct ApiRange {
  explicit ApiRange(const char *name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange &) = delete;
  ApiRange &operator=(const ApiRange &) = delete;
};

unsigned *error_word_ptr() {
  // the device address of g_error_word on the current device
  static thread_local int cached_dev = -1;
  static thread_local unsigned *cached = nullptr;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != cached_dev) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    cached = (unsigned *)p;
    cached_dev = dev;
  }
  return cached;
}

// validates one codec; fills the internal bundle
static int check_codec(const nanokv_codec *c, const char *name, bool need_E, Codec *out) {
  if (!c) return fail(NANOKV_ERR_INVALID, "%s: codec is NULL", name);
  if (c->H < 1 || c->H > 256) return fail(NANOKV_ERR_INVALID, "%s: H=%d out of range [1,256]", name, c->H);
  if (!(c->d == 16 || c->d == 32 || c->d == 64 || c->d == 128))
    return fail(NANOKV_ERR_UNSUPPORTED, "%s: d=%d (supported: 16, 32, 64, 128)", name, c->d);
  if (c->r < 2 || c->r > 512 || (c->r & 1))
    return fail(NANOKV_ERR_INVALID, "%s: r=%d must be even and in [2,512]", name, c->r);
  if (c->C < 1 || c->C > 256) return fail(NANOKV_ERR_INVALID, "%s: C=%d out of range [1,256]", name, c->C);
  int prec;
  if (c->param_dtype == NANOKV_F32 && c->scale_dtype == NANOKV_F32) prec = PREC_F32;
  else if (c->param_dtype == NANOKV_BF16 && c->scale_dtype == NANOKV_F16) prec = PREC_BF16;
  else
    return fail(NANOKV_ERR_UNSUPPORTED,
                "%s: param/scale dtype pair (%d,%d) unsupported (F32/F32 or BF16/F16)", name,
                c->param_dtype, c->scale_dtype);
  if (!c->centers || !c->D || (need_E && !c->E))
    return fail(NANOKV_ERR_INVALID, "%s: NULL parameter pointer", name);
  if (!aligned16(c->centers) || !aligned16(c->D) || (c->E && !aligned16(c->E)))
    return fail(NANOKV_ERR_INVALID, "%s: parameter pointers must be 16-byte aligned", name);
  if (c->aux && !aligned16(c->aux))
    return fail(NANOKV_ERR_INVALID, "%s: aux must be 16-byte aligned", name);
  *out = Codec{c->H, c->d, c->r, c->C, prec, c->centers, c->D, c->E, c->aux};
  return NANOKV_OK;
}

static int io_prec(int32_t dt) {
  if (dt == NANOKV_F32) return PREC_F32;
  if (dt == NANOKV_BF16) return PREC_BF16;
  return -1;
}

// Tokens attended on the full-dim path.  The low-dim and full-dim paths give
// the same attention over the same compressed tokens (the low-dim form only
// reorders the contraction), so when the tensor-core kernels have no low-dim
// kernel for a codec shape but do have the full-dim one, the low-dim tokens
// are attended there too (paths 0 and 2); path 1 keeps the routing as given.
static int64_t effective_T_full(int path, bool tc_low_ok, bool tc_full_ok, int64_t T, int64_t T_full) {
  if (path != 1 && T > T_full && !tc_low_ok && tc_full_ok) return T;
  return T_full;
}

// a low-dim tensor-core kernel exists for these codecs: the single-CTA one
// (r <= 192, C <= 64) or the 2-CTA one for larger codecs
static bool tc_low_any(const Codec &ck, const Codec &cv) {
  return tc_low_supported(ck, cv) || tc_low_pair_supported(ck, cv);
}

// workspace carve-up (every region 256-byte aligned)
struct WsLayout {
  // branch b (0 low-dim, 1 full-dim, 2 current chunk) has nparts[b]
  // consecutive partials, osz / lsz bytes apart
  size_t off_O[3], off_L[3], off_qred, off_qc, total, osz, lsz;
  int nparts[3];
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

static WsLayout ws_layout(int64_t Tq, const Codec &ck, int64_t T_low, int64_t T_full,
                          int64_t T_cur, bool tc_low, int full_splits) {
  WsLayout w{};
  size_t off = 0;
  w.osz = al256((size_t)Tq * ck.H * ck.d * sizeof(float));
  w.lsz = al256((size_t)Tq * ck.H * sizeof(float));
  const bool on[3] = {T_low > 0, T_full > 0, T_cur > 0};
  for (int b = 0; b < 3; ++b) {
    w.nparts[b] = on[b] ? (b == 1 ? full_splits : 1) : 0;
    w.off_O[b] = off;
    off += w.nparts[b] * w.osz;
    w.off_L[b] = off;
    off += w.nparts[b] * w.lsz;
  }
  w.off_qred = w.off_qc = off;
  if (T_low > 0 && !tc_low) {
    w.off_qred = off;
    off += al256((size_t)ck.H * Tq * ck.r * sizeof(float));
    w.off_qc = off;
    off += al256((size_t)ck.H * Tq * ck.C * sizeof(float));
  }
  w.total = off;
  return w;
}

// ---------------------------------------------------------------------------
// routed attend: a full-dim routing policy given as token ranges and heads
// ---------------------------------------------------------------------------
struct RoutedPlan {
  int64_t T_f = 0, T_l = 0;  // history tokens read full-dim / low-dim (ordinary heads)
  GatherSegs full{}, low{};  // segments of the two sets
  uint8_t cls[256] = {};     // HeadClass of each head's low-dim tokens
  int ncls[HC_COUNT] = {};   // heads per class
  int nred = 0;              // heads at a reduced attention dimension
  HeadDims dims{};
  // workspace: gathered histories [set][branch] (ids, codes, scales), head
  // lists, reduced queries
  size_t off_ids[2][2], off_codes[2][2], off_scales[2][2], off_heads, off_qred, total;
};

static bool lowdim_codecs_ok(const Codec &ck, const Codec &cv) {
  return ck.prec == PREC_BF16 && cv.prec == PREC_BF16 && ck.d == 128 && cv.d == 128 && ck.H == cv.H &&
         ck.r == cv.r;
}

static int routed_plan(const Codec &ck, const Codec &cv, int64_t Tq, int64_t T, const nanokv_range *full,
                       int32_t n_full, const uint8_t *full_heads, const nanokv_lowdim *lowdim, size_t base,
                       RoutedPlan *p) {
  if (n_full < 0 || n_full > NANOKV_MAX_RANGES)
    return fail(NANOKV_ERR_INVALID, "routed: n_full=%d out of range [0,%d]", n_full, NANOKV_MAX_RANGES);
  if (n_full > 0 && !full) return fail(NANOKV_ERR_INVALID, "routed: NULL range array with n_full > 0");
  RoutedPlan r;
  int64_t prev_end = 0;
  for (int i = 0; i < n_full; ++i) {
    const int64_t s0 = full[i].start, c = full[i].count;
    if (s0 < prev_end || c < 0 || s0 + c > T)
      return fail(NANOKV_ERR_INVALID, "routed: range %d [%lld, +%lld) not sorted, disjoint and inside [0, %lld)", i,
                  (long long)s0, (long long)c, (long long)T);
    if (c > 0) {
      if (s0 > prev_end) {  // the gap before this range is low-dim
        r.low.src[r.low.n] = prev_end;
        r.low.dst[r.low.n] = r.T_l;
        r.low.cnt[r.low.n++] = s0 - prev_end;
        r.T_l += s0 - prev_end;
      }
      r.full.src[r.full.n] = s0;
      r.full.dst[r.full.n] = r.T_f;
      r.full.cnt[r.full.n++] = c;
      r.T_f += c;
      prev_end = s0 + c;
    }
  }
  if (T > prev_end) {
    r.low.src[r.low.n] = prev_end;
    r.low.dst[r.low.n] = r.T_l;
    r.low.cnt[r.low.n++] = T - prev_end;
    r.T_l += T - prev_end;
  }
  if (lowdim && !lowdim->d_h) return fail(NANOKV_ERR_INVALID, "routed: lowdim given with a NULL d_h array");
  for (int h = 0; h < ck.H; ++h) {
    const int dh = lowdim ? lowdim->d_h[h] : 0;
    if (!(dh == 0 || tc_reduced_dim_ok(dh)))
      return fail(NANOKV_ERR_INVALID, "routed: d_h[%d]=%d (0, 32, 64 or 96; full 128 goes in full_heads)", h, dh);
    uint8_t c = HC_LOW;
    if (full_heads && full_heads[h]) c = HC_FULL;
    else if (dh) {
      c = dh == 32 ? HC_R32 : dh == 64 ? HC_R64 : HC_R96;
      r.dims.d[h] = (uint8_t)dh;
      ++r.nred;
    }
    r.cls[h] = c;
    ++r.ncls[c];
  }
  if (r.nred > 0) {
    if (!lowdim_codecs_ok(ck, cv))
      return fail(NANOKV_ERR_UNSUPPORTED, "routed: reduced attention dimensions need bf16 codecs with d = 128");
    if (!lowdim->U || !lowdim->W || !lowdim->aux || !aligned16(lowdim->U) || !aligned16(lowdim->W) ||
        !aligned16(lowdim->aux))
      return fail(NANOKV_ERR_INVALID, "routed: lowdim U, W and aux must be non-NULL and 16-byte aligned");
  }
  // gathered histories, then the head lists, then the reduced queries
  size_t off = base;
  const int64_t n[2] = {r.T_f, r.T_l};
  const Codec *c[2] = {&ck, &cv};
  const size_t sb = ck.prec == PREC_F32 ? 4 : 2;
  for (int set = 0; set < 2; ++set)
    for (int br = 0; br < 2; ++br) {
      r.off_ids[set][br] = off;
      off += al256((size_t)n[set]);
      r.off_codes[set][br] = off;
      off += al256((size_t)n[set] * (c[br]->r / 2));
      r.off_scales[set][br] = off;
      off += al256((size_t)n[set] * sb);
    }
  r.off_heads = off;
  off += al256((size_t)(HC_COUNT + 1) * ck.H * sizeof(int32_t));
  r.off_qred = off;
  if (r.nred > 0 && r.T_l > 0) off += al256((size_t)Tq * ck.H * 128 * 2);
  r.total = off;
  *p = r;
  return NANOKV_OK;
}

}  // namespace nanokv

using namespace nanokv;

extern "C" {

const char *nanokv_last_error(void) { return t_last_error.c_str(); }

const char *nanokv_version(void) { return "nanokv-b200 0.1 (sm_100a)"; }

int nanokv_set_kernel_path(int32_t path) {
  if (path < 0 || path > 2) return -1;
  return g_kernel_path.exchange(path);
}

int nanokv_check(void *stream) {
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_status(e, "stream");
  unsigned *p = error_word_ptr();
  if (!p) return fail(NANOKV_ERR_CUDA, "cannot resolve the device error word");
  unsigned w = 0;
  e = cudaMemcpy(&w, p, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e, "read error word");
  if (w) {
    const unsigned zero = 0;
    cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (w & ERRW_TIMEOUT) return fail(NANOKV_ERR_TIMEOUT, "a kernel gave up on a bounded wait (word 0x%x)", w);
    return fail(NANOKV_ERR_CUDA, "device error word 0x%x", w);
  }
  return NANOKV_OK;
}

int64_t nanokv_attend_full_tokens(const nanokv_codec *ck, const nanokv_codec *cv, int64_t T, int64_t T_full) {
  Codec a, b;
  if (T < 0 || T_full < 0 || T_full > T) return -1;
  if (check_codec(ck, "ck", false, &a) || check_codec(cv, "cv", false, &b)) return -1;
  return effective_T_full(g_kernel_path.load(), tc_low_any(a, b), tc_full_supported(a, b), T, T_full);
}

int nanokv_selftest_wait(uint64_t limit_ns, void *stream) {
  const uint64_t lim = limit_ns < 1000000ull ? 1000000ull : (limit_ns > 2000000000ull ? 2000000000ull : limit_ns);
  unsigned *errw = error_word_ptr();
  if (!errw) return fail(NANOKV_ERR_CUDA, "cannot resolve the device error word");
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(lim, errw);
  return cuda_status(cudaGetLastError(), "selftest launch");
}

int nanokv_encode(const nanokv_codec *ck, const nanokv_codec *cv, const void *k, const void *v,
                  int32_t x_dtype, int64_t T, uint8_t *ids_k, uint8_t *codes_k, void *scales_k,
                  uint8_t *ids_v, uint8_t *codes_v, void *scales_v, void *stream) {
  ApiRange range("nanokv_encode");
  if (T < 0) return fail(NANOKV_ERR_INVALID, "encode: T=%lld < 0", (long long)T);
  if (!ck && !cv) return fail(NANOKV_ERR_INVALID, "encode: both codecs are NULL");
  Codec c[2];
  const nanokv_codec *in[2] = {ck, cv};
  const void *x[2] = {k, v};
  uint8_t *ids[2] = {ids_k, ids_v};
  uint8_t *codes[2] = {codes_k, codes_v};
  void *scales[2] = {scales_k, scales_v};
  const int xp = io_prec(x_dtype);
  for (int b = 0; b < 2; ++b) {
    if (!in[b]) continue;
    int s = check_codec(in[b], b ? "encode cv" : "encode ck", true, &c[b]);
    if (s) return s;
    if (xp != c[b].prec) return fail(NANOKV_ERR_UNSUPPORTED, "encode: x_dtype must equal param_dtype");
    if (T > 0 && (!x[b] || !ids[b] || !codes[b] || !scales[b]))
      return fail(NANOKV_ERR_INVALID, "encode: NULL input/output pointer for branch %d", b);
    if (T > 0 && (!aligned16(x[b]) || !aligned16(codes[b])))
      return fail(NANOKV_ERR_INVALID, "encode: pointers must be 16-byte aligned");
  }
  if (T == 0) return NANOKV_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const int path = g_kernel_path.load();
  bool tc_ok[2] = {false, false};
  for (int b = 0; b < 2; ++b) {
    if (!in[b]) continue;
    tc_ok[b] = tc_encode_supported(c[b]);
    if (path == 2 && !tc_ok[b])
      return fail(NANOKV_ERR_UNSUPPORTED, "encode: no tensor-core kernel for this shape (or codec aux missing)");
  }
  // both branches in one tensor-core launch when their shapes agree
  if (path != 1 && in[0] && in[1] && tc_ok[0] && tc_ok[1] && c[0].C == c[1].C && c[0].r == c[1].r) {
    cudaError_t e = timed(NANOKV_K_ENCODE, 1, st, [&] {
      return tc_encode_pair(c, x, T, ids, codes, scales, 2, st);
    });
    return cuda_status(e, "encode launch");
  }
  for (int b = 0; b < 2; ++b) {
    if (!in[b]) continue;
    cudaError_t e = timed(NANOKV_K_ENCODE, 1, st, [&] {
      return (path != 1 && tc_ok[b]) ? tc_encode_pair(&c[b], &x[b], T, &ids[b], &codes[b], &scales[b], 1, st)
                                     : simt_encode(c[b], x[b], T, ids[b], codes[b], scales[b], st);
    });
    if (e != cudaSuccess) return cuda_status(e, "encode launch");
  }
  return NANOKV_OK;
}

size_t nanokv_codec_aux_bytes(const nanokv_codec *c_) {
  Codec c;
  if (check_codec(c_, "codec", false, &c)) return 0;
  return codec_aux_bytes(c);
}

int nanokv_codec_prepare(const nanokv_codec *c_, void *aux, void *stream) {
  ApiRange range("nanokv_codec_prepare");
  Codec c;
  int s = check_codec(c_, "prepare", true, &c);
  if (s) return s;
  if (!aux || !aligned16(aux)) return fail(NANOKV_ERR_INVALID, "prepare: aux NULL or misaligned");
  return cuda_status(codec_prepare(c, aux, (cudaStream_t)stream), "prepare launch");
}

size_t nanokv_attend_workspace(int64_t Tq, const nanokv_codec *ck, const nanokv_codec *cv,
                               int64_t T, int64_t T_full, int64_t T_cur) {
  Codec a, b;
  if (Tq < 0 || T < 0 || T_full < 0 || T_full > T || T_cur < 0) return 0;
  if (check_codec(ck, "ck", false, &a) || check_codec(cv, "cv", false, &b)) return 0;
  const int path = g_kernel_path.load();
  const bool tc_low = path != 1 && tc_low_any(a, b);
  const bool tc_full = path != 1 && tc_full_supported(a, b);
  T_full = effective_T_full(path, tc_low_any(a, b), tc_full_supported(a, b), T, T_full);
  const int splits = (tc_full && T_full > 0 && Tq > 0) ? tc_full_splits(Tq, a.H, a.d, T_full) : 1;
  return ws_layout(Tq, a, T - T_full, T_full, T_cur, tc_low, splits).total;
}

// nanokv_attend, with its output in the codecs' precision (out_f32 false) or
// in fp32 (nanokv_attend_partial)
static int attend_impl(const void *q, int32_t io_dtype, int64_t Tq, const nanokv_codec *ck_,
                       const nanokv_codec *cv_, const nanokv_hist *hk_, const nanokv_hist *hv_, int64_t T,
                       int64_t T_full, const void *k_cur, const void *v_cur, int64_t T_cur, float softmax_scale,
                       void *out, float *lse_out, void *workspace, size_t workspace_bytes, void *stream,
                       bool out_f32) {
  Codec ck, cv;
  int s;
  if ((s = check_codec(ck_, "attend ck", false, &ck))) return s;
  if ((s = check_codec(cv_, "attend cv", false, &cv))) return s;
  if (ck.H != cv.H || ck.d != cv.d || ck.prec != cv.prec)
    return fail(NANOKV_ERR_INVALID, "attend: ck and cv must share H, d and dtypes");
  const int iop = io_prec(io_dtype);
  if (iop != ck.prec) return fail(NANOKV_ERR_UNSUPPORTED, "attend: io_dtype must equal param_dtype");
  if (Tq < 0 || T < 0 || T_cur < 0 || T_full < 0 || T_full > T)
    return fail(NANOKV_ERR_INVALID, "attend: bad sizes Tq=%lld T=%lld T_full=%lld T_cur=%lld",
                (long long)Tq, (long long)T, (long long)T_full, (long long)T_cur);
  if (!(softmax_scale == softmax_scale) || softmax_scale <= 0.f || softmax_scale > 1e4f)
    return fail(NANOKV_ERR_INVALID, "attend: softmax_scale must be finite and positive");
  if (Tq == 0) return NANOKV_OK;
  if (!q || !out) return fail(NANOKV_ERR_INVALID, "attend: NULL q or out");
  if (!aligned16(q) || !aligned16(out) || (lse_out && !aligned16(lse_out)))
    return fail(NANOKV_ERR_INVALID, "attend: q/out/lse_out must be 16-byte aligned");
  if (T > 0) {
    if (!hk_ || !hv_ || !hk_->ids || !hk_->codes || !hk_->scales || !hv_->ids || !hv_->codes ||
        !hv_->scales)
      return fail(NANOKV_ERR_INVALID, "attend: NULL history pointer with T > 0");
    if (!aligned16(hk_->codes) || !aligned16(hv_->codes))
      return fail(NANOKV_ERR_INVALID, "attend: code pointers must be 16-byte aligned");
  }
  if (T_cur > 0 && (!k_cur || !v_cur || !aligned16(k_cur) || !aligned16(v_cur)))
    return fail(NANOKV_ERR_INVALID, "attend: k_cur/v_cur NULL or misaligned with T_cur > 0");

  const int path = g_kernel_path.load();
  const bool tc_full_ok = tc_full_supported(ck, cv);
  const bool tc_low_ok = tc_low_any(ck, cv);
  T_full = effective_T_full(path, tc_low_ok, tc_full_ok, T, T_full);
  const int64_t T_low = T - T_full;
  const bool tc_dense_ok = tc_dense_supported(ck.prec, ck.d);
  if (path == 2 && ((T_full > 0 && !tc_full_ok) || (T_low > 0 && !tc_low_ok) ||
                    (T_cur > 0 && !tc_dense_ok)))
    return fail(NANOKV_ERR_UNSUPPORTED, "attend: no tensor-core kernel for this shape");
  const bool use_tc_low = path != 1 && tc_low_ok;
  const bool use_tc_full = path != 1 && tc_full_ok;
  const int full_splits = (use_tc_full && T_full > 0) ? tc_full_splits(Tq, ck.H, ck.d, T_full) : 1;
  const WsLayout w = ws_layout(Tq, ck, T_low, T_full, T_cur, use_tc_low, full_splits);
  if (w.total > 0 && (!workspace || workspace_bytes < w.total))
    return fail(NANOKV_ERR_INVALID, "attend: workspace needs %zu bytes, got %zu", w.total,
                workspace_bytes);
  if (workspace && !aligned16(workspace))
    return fail(NANOKV_ERR_INVALID, "attend: workspace must be 16-byte aligned");

  cudaStream_t st = (cudaStream_t)stream;
  char *ws = (char *)workspace;
  const Hist hk = T > 0 ? Hist{hk_->ids, hk_->codes, hk_->scales} : Hist{};
  const Hist hv = T > 0 ? Hist{hv_->ids, hv_->codes, hv_->scales} : Hist{};
  PartList pl{};
  cudaError_t e = cudaSuccess;
  const bool on[3] = {T_low > 0, T_full > 0, T_cur > 0};
  const int nbranch = (int)on[0] + (int)on[1] + (int)on[2];
  // one branch: everything on the caller's stream; several: fork onto the
  // helper streams after the caller's prior work, join before the merge.
  // With per-kernel timing on, the branches run one after another on the
  // caller's stream, so that each kernel's events time it alone.
  std::unique_lock<std::mutex> lk(g_bs_mu, std::defer_lock);
  BranchStreams *bs = nullptr;
  if (nbranch > 1 && !g_timing.load()) {
    lk.lock();
    if ((e = branch_streams(&bs)) != cudaSuccess) return cuda_status(e, "attend helper streams");
    if ((e = cudaEventRecord(bs->fork, st)) != cudaSuccess) return cuda_status(e, "attend fork");
  }
  auto bstream = [&](int b) -> cudaStream_t {
    if (!bs) return st;
    e = cudaStreamWaitEvent(bs->s[b], bs->fork, 0);
    return bs->s[b];
  };
  auto join = [&](int b) -> cudaError_t {
    if (!bs) return cudaSuccess;
    cudaError_t e2 = cudaEventRecord(bs->join[b], bs->s[b]);
    return e2 == cudaSuccess ? cudaStreamWaitEvent(st, bs->join[b], 0) : e2;
  };
  if (on[0]) {
    Part p{(float *)(ws + w.off_O[0]), (float *)(ws + w.off_L[0])};
    cudaStream_t bst = bstream(0);
    if (e != cudaSuccess) return cuda_status(e, "attend fork");
    if (use_tc_low) {
      e = timed(NANOKV_K_LOW, 1, bst, [&] {
        return tc_low_supported(ck, cv) ? tc_attend_low(q, Tq, ck, cv, hk, hv, 0, T_low, softmax_scale, p, bst)
                                        : tc_attend_low_pair(q, Tq, ck, cv, hk, hv, 0, T_low, softmax_scale, p, bst);
      });
    } else {
      float *qred = (float *)(ws + w.off_qred), *qc = (float *)(ws + w.off_qc);
      e = timed(NANOKV_K_LOW, 2, bst, [&] {
        cudaError_t e2 = simt_low_prep(q, Tq, ck, qred, qc, bst);
        if (e2 == cudaSuccess)
          e2 = simt_attend_low(qred, qc, Tq, ck, cv, hk, hv, 0, T_low, softmax_scale, p, bst);
        return e2;
      });
    }
    if (e == cudaSuccess) e = join(0);
    if (e != cudaSuccess) return cuda_status(e, "attend low-dim launch");
    pl.O[pl.n] = p.O;
    pl.LSE[pl.n++] = p.LSE;
  }
  if (on[1]) {
    Part p{(float *)(ws + w.off_O[1]), (float *)(ws + w.off_L[1])};
    cudaStream_t bst = bstream(1);
    if (e != cudaSuccess) return cuda_status(e, "attend fork");
    e = timed(NANOKV_K_FULL, 1, bst, [&] {
      return use_tc_full ? tc_attend_full(q, Tq, ck, cv, hk, hv, T_low, T_full, softmax_scale, p, full_splits,
                                          w.osz / sizeof(float), w.lsz / sizeof(float), bst, false)
                         : simt_attend_full(q, Tq, ck, cv, hk, hv, T_low, T_full, softmax_scale, p, bst);
    });
    if (e == cudaSuccess) e = join(1);
    if (e != cudaSuccess) return cuda_status(e, "attend full-dim launch");
    for (int z = 0; z < w.nparts[1]; ++z) {
      pl.O[pl.n] = (const float *)(ws + w.off_O[1] + z * w.osz);
      pl.LSE[pl.n++] = (const float *)(ws + w.off_L[1] + z * w.lsz);
    }
  }
  if (on[2]) {
    Part p{(float *)(ws + w.off_O[2]), (float *)(ws + w.off_L[2])};
    cudaStream_t bst = bstream(2);
    if (e != cudaSuccess) return cuda_status(e, "attend fork");
    e = timed(NANOKV_K_DENSE, 1, bst, [&] {
      return (path != 1 && tc_dense_ok)
                 ? tc_attend_dense(q, Tq, ck.H, ck.d, k_cur, v_cur, T_cur, softmax_scale, p, bst, false)
                 : simt_attend_dense(ck.prec, q, Tq, ck.H, ck.d, k_cur, v_cur, T_cur,
                                     softmax_scale, p, bst);
    });
    if (e == cudaSuccess) e = join(2);
    if (e != cudaSuccess) return cuda_status(e, "attend current-chunk launch");
    pl.O[pl.n] = p.O;
    pl.LSE[pl.n++] = p.LSE;
  }
  if (lk.owns_lock()) lk.unlock();
  e = timed(NANOKV_K_MERGE, 1, st,
            [&] { return lse_merge_launch(pl, Tq, ck.H, ck.d, out, out_f32 ? (int)PREC_F32 : ck.prec, lse_out, st); });
  return cuda_status(e, "attend merge launch");
}

int nanokv_attend(const void *q, int32_t io_dtype, int64_t Tq, const nanokv_codec *ck_,
                  const nanokv_codec *cv_, const nanokv_hist *hk_, const nanokv_hist *hv_,
                  int64_t T, int64_t T_full, const void *k_cur, const void *v_cur, int64_t T_cur,
                  float softmax_scale, void *out, float *lse_out, void *workspace,
                  size_t workspace_bytes, void *stream) {
  ApiRange range("nanokv_attend");
  return attend_impl(q, io_dtype, Tq, ck_, cv_, hk_, hv_, T, T_full, k_cur, v_cur, T_cur, softmax_scale, out,
                     lse_out, workspace, workspace_bytes, stream, false);
}

int nanokv_attend_partial(const void *q, int32_t io_dtype, int64_t Tq, const nanokv_codec *ck_,
                          const nanokv_codec *cv_, const nanokv_hist *hk_, const nanokv_hist *hv_, int64_t T,
                          int64_t T_full, const void *k_cur, const void *v_cur, int64_t T_cur,
                          float softmax_scale, float *out, float *lse_out, void *workspace,
                          size_t workspace_bytes, void *stream) {
  ApiRange range("nanokv_attend_partial");
  if (Tq > 0 && !lse_out) return fail(NANOKV_ERR_INVALID, "attend_partial: lse_out is required");
  return attend_impl(q, io_dtype, Tq, ck_, cv_, hk_, hv_, T, T_full, k_cur, v_cur, T_cur, softmax_scale, out,
                     lse_out, workspace, workspace_bytes, stream, true);
}

// How a routed call runs its two history sets.  `full_set`: the routed
// tokens, all heads, full-dim.  `low_set`, per head class: the heads kept
// full-dim on the full-dim kernel; the ordinary heads on the low-dim kernel
// (tensor-core or CUDA-core), or on the tensor-core full-dim kernel where no
// low-dim one exists (as in nanokv_attend); the reduced heads on the full-dim
// kernel at their width.  `cls` / `ncls`: the classes after that choice.
struct RoutedKernels {
  bool tc_full, tc_low, tc_dense, low_via_full, low_simt;
  uint8_t cls[256];
  int ncls[HC_COUNT];
};

static int routed_kernels(int path, const Codec &ck, const Codec &cv, const RoutedPlan &r, int64_t T_cur,
                          RoutedKernels *k) {
  const bool full_ok = tc_full_supported(ck, cv), low_ok = tc_low_any(ck, cv);
  k->tc_full = path != 1 && full_ok;
  k->tc_low = path != 1 && low_ok;
  k->tc_dense = path != 1 && tc_dense_supported(ck.prec, ck.d);
  k->low_via_full = !k->tc_low && k->tc_full;
  const int nlow = r.ncls[HC_LOW];
  k->low_simt = r.T_l > 0 && nlow > 0 && !k->tc_low && !k->low_via_full;
  if (path == 2 && ((r.T_f > 0 && !k->tc_full) || (r.T_l > 0 && nlow > 0 && !k->tc_low && !k->low_via_full) ||
                    (T_cur > 0 && !k->tc_dense)))
    return fail(NANOKV_ERR_UNSUPPORTED, "routed: no tensor-core kernel for this shape");
  if (r.T_l > 0 && r.nred > 0 && !k->tc_full)
    return fail(NANOKV_ERR_UNSUPPORTED, "routed: reduced attention dimensions need the tensor-core kernels");
  for (int c = 0; c < HC_COUNT; ++c) k->ncls[c] = 0;
  for (int h = 0; h < ck.H; ++h) {
    k->cls[h] = (r.cls[h] == HC_LOW && k->low_via_full) ? (uint8_t)HC_FULL : r.cls[h];
    ++k->ncls[k->cls[h]];
  }
  int present = 0;
  for (int c = 0; c < HC_COUNT; ++c) present += k->ncls[c] > 0;
  // a launch over part of the heads needs a kernel that takes a head list
  if (r.T_l > 0 && present > 1 &&
      ((k->ncls[HC_FULL] > 0 && !k->tc_full) || (k->ncls[HC_LOW] > 0 && !k->tc_low)))
    return fail(NANOKV_ERR_UNSUPPORTED,
                "routed: heads of several kinds in one call need the tensor-core kernels for this codec");
  return NANOKV_OK;
}

size_t nanokv_attend_routed_workspace(int64_t Tq, const nanokv_codec *ck_, const nanokv_codec *cv_, int64_t T,
                                      const nanokv_range *full, int32_t n_full, const uint8_t *full_heads,
                                      const nanokv_lowdim *lowdim, int64_t T_cur) {
  Codec ck, cv;
  if (Tq < 0 || T < 0 || T_cur < 0) return 0;
  if (check_codec(ck_, "ck", false, &ck) || check_codec(cv_, "cv", false, &cv)) return 0;
  RoutedPlan r;
  if (routed_plan(ck, cv, Tq, T, full, n_full, full_heads, lowdim, 0, &r)) return 0;
  RoutedKernels k;
  if (routed_kernels(g_kernel_path.load(), ck, cv, r, T_cur, &k)) return 0;
  const int splits = (k.tc_full && r.T_f > 0 && Tq > 0) ? tc_full_splits(Tq, ck.H, ck.d, r.T_f) : 1;
  const WsLayout w = ws_layout(Tq, ck, r.T_l, r.T_f, T_cur, !k.low_simt, splits);
  RoutedPlan r2;
  routed_plan(ck, cv, Tq, T, full, n_full, full_heads, lowdim, w.total, &r2);
  return r2.total;
}

int nanokv_attend_routed(const void *q, int32_t io_dtype, int64_t Tq, const nanokv_codec *ck_,
                         const nanokv_codec *cv_, const nanokv_hist *hk_, const nanokv_hist *hv_, int64_t T,
                         const nanokv_range *full, int32_t n_full, const uint8_t *full_heads,
                         const nanokv_lowdim *lowdim, const void *k_cur, const void *v_cur, int64_t T_cur,
                         float softmax_scale, void *out, float *lse_out, void *workspace, size_t workspace_bytes,
                         void *stream) {
  ApiRange range("nanokv_attend_routed");
  Codec ck, cv;
  int s;
  if ((s = check_codec(ck_, "routed ck", false, &ck))) return s;
  if ((s = check_codec(cv_, "routed cv", false, &cv))) return s;
  if (ck.H != cv.H || ck.d != cv.d || ck.prec != cv.prec)
    return fail(NANOKV_ERR_INVALID, "routed: ck and cv must share H, d and dtypes");
  if (io_prec(io_dtype) != ck.prec) return fail(NANOKV_ERR_UNSUPPORTED, "routed: io_dtype must equal param_dtype");
  if (Tq < 0 || T < 0 || T_cur < 0)
    return fail(NANOKV_ERR_INVALID, "routed: bad sizes Tq=%lld T=%lld T_cur=%lld", (long long)Tq, (long long)T,
                (long long)T_cur);
  if (!(softmax_scale == softmax_scale) || softmax_scale <= 0.f || softmax_scale > 1e4f)
    return fail(NANOKV_ERR_INVALID, "routed: softmax_scale must be finite and positive");
  RoutedPlan r;
  if ((s = routed_plan(ck, cv, Tq, T, full, n_full, full_heads, lowdim, 0, &r))) return s;
  if (Tq == 0) return NANOKV_OK;
  if (!q || !out) return fail(NANOKV_ERR_INVALID, "routed: NULL q or out");
  if (!aligned16(q) || !aligned16(out) || (lse_out && !aligned16(lse_out)))
    return fail(NANOKV_ERR_INVALID, "routed: q/out/lse_out must be 16-byte aligned");
  if (T > 0 && (!hk_ || !hv_ || !hk_->ids || !hk_->codes || !hk_->scales || !hv_->ids || !hv_->codes || !hv_->scales))
    return fail(NANOKV_ERR_INVALID, "routed: NULL history pointer with T > 0");
  if (T_cur > 0 && (!k_cur || !v_cur || !aligned16(k_cur) || !aligned16(v_cur)))
    return fail(NANOKV_ERR_INVALID, "routed: k_cur/v_cur NULL or misaligned with T_cur > 0");
  const int path = g_kernel_path.load();
  RoutedKernels k;
  if ((s = routed_kernels(path, ck, cv, r, T_cur, &k))) return s;
  const int splits = (k.tc_full && r.T_f > 0) ? tc_full_splits(Tq, ck.H, ck.d, r.T_f) : 1;
  const WsLayout w = ws_layout(Tq, ck, r.T_l, r.T_f, T_cur, !k.low_simt, splits);
  routed_plan(ck, cv, Tq, T, full, n_full, full_heads, lowdim, w.total, &r);
  if (r.total > 0 && (!workspace || workspace_bytes < r.total))
    return fail(NANOKV_ERR_INVALID, "routed: workspace needs %zu bytes, got %zu", r.total, workspace_bytes);
  if (workspace && !aligned16(workspace)) return fail(NANOKV_ERR_INVALID, "routed: workspace must be 16-byte aligned");

  cudaStream_t st = (cudaStream_t)stream;
  char *ws = (char *)workspace;
  cudaError_t e = cudaSuccess;
  // 1. gather the two sets (and the head lists) into the workspace
  Hist hs[2][2];  // [set][branch]
  const int sb = ck.prec == PREC_F32 ? 4 : 2;
  if (T > 0) {
    GatherArgs g{};
    const nanokv_hist *src[2] = {hk_, hv_};
    const Codec *c[2] = {&ck, &cv};
    for (int br = 0; br < 2; ++br) {
      g.ids[br] = src[br]->ids;
      g.codes[br] = src[br]->codes;
      g.scales[br] = (const uint8_t *)src[br]->scales;
      g.row_bytes[br] = c[br]->r / 2;
      for (int set = 0; set < 2; ++set) {
        g.d_ids[set][br] = (uint8_t *)(ws + r.off_ids[set][br]);
        g.d_codes[set][br] = (uint8_t *)(ws + r.off_codes[set][br]);
        g.d_scales[set][br] = (uint8_t *)(ws + r.off_scales[set][br]);
        hs[set][br] = Hist{g.d_ids[set][br], g.d_codes[set][br], g.d_scales[set][br]};
      }
    }
    g.n_out[0] = r.T_f;
    g.n_out[1] = r.T_l;
    g.scale_bytes = sb;
    for (int h = 0; h < ck.H; ++h) g.head_class[h] = k.cls[h];
    g.H = ck.H;
    g.head_lists = (int32_t *)(ws + r.off_heads);
    if ((e = gather_launch(r.full, r.low, g, st)) != cudaSuccess) return cuda_status(e, "routed gather launch");
  }
  const int32_t *lists = (const int32_t *)(ws + r.off_heads);
  // the heads of class c: all heads (no list) when the class holds every head
  auto sel = [&](int c) {
    return k.ncls[c] == ck.H ? HeadSel{nullptr, 0} : HeadSel{lists + (size_t)c * ck.H, k.ncls[c]};
  };

  // 2. branches: routed tokens full-dim (all heads); the other tokens low-dim
  // for the ordinary heads and full-dim for the heads kept full; the current
  // chunk.  Independent: on the helper streams, as in nanokv_attend.
  PartList pl{};
  const bool on[3] = {r.T_l > 0, r.T_f > 0, T_cur > 0};
  const int nbranch = (int)on[0] + (int)on[1] + (int)on[2] + (int)(on[0] && r.nred > 0);
  std::unique_lock<std::mutex> lk(g_bs_mu, std::defer_lock);
  BranchStreams *bs = nullptr;
  if (nbranch > 1 && !g_timing.load()) {
    lk.lock();
    if ((e = branch_streams(&bs)) != cudaSuccess) return cuda_status(e, "routed helper streams");
    if ((e = cudaEventRecord(bs->fork, st)) != cudaSuccess) return cuda_status(e, "routed fork");
  }
  auto bstream = [&](int b) -> cudaStream_t {
    if (!bs) return st;
    e = cudaStreamWaitEvent(bs->s[b], bs->fork, 0);
    return bs->s[b];
  };
  auto join = [&](int b) -> cudaError_t {
    if (!bs) return cudaSuccess;
    cudaError_t e2 = cudaEventRecord(bs->join[b], bs->s[b]);
    return e2 == cudaSuccess ? cudaStreamWaitEvent(st, bs->join[b], 0) : e2;
  };
  if (on[0]) {
    Part p{(float *)(ws + w.off_O[0]), (float *)(ws + w.off_L[0])};
    cudaStream_t bst = bstream(0);
    if (e != cudaSuccess) return cuda_status(e, "routed fork");
    const Hist &lk_ = hs[1][0], &lv_ = hs[1][1];
    // each head class into the same partial (disjoint heads)
    if (k.ncls[HC_FULL]) {
      e = timed(NANOKV_K_FULL, 1, bst, [&] {
        return k.tc_full ? tc_attend_full(q, Tq, ck, cv, lk_, lv_, 0, r.T_l, softmax_scale, p, 1, 0, 0, bst, false,
                                          sel(HC_FULL))
                         : simt_attend_full(q, Tq, ck, cv, lk_, lv_, 0, r.T_l, softmax_scale, p, bst);
      });
    }
    if (e == cudaSuccess && k.ncls[HC_LOW]) {
      if (k.tc_low) {
        e = timed(NANOKV_K_LOW, 1, bst, [&] {
          return tc_low_supported(ck, cv)
                     ? tc_attend_low(q, Tq, ck, cv, lk_, lv_, 0, r.T_l, softmax_scale, p, bst, sel(HC_LOW))
                     : tc_attend_low_pair(q, Tq, ck, cv, lk_, lv_, 0, r.T_l, softmax_scale, p, bst, sel(HC_LOW));
        });
      } else {
        float *qred = (float *)(ws + w.off_qred), *qc = (float *)(ws + w.off_qc);
        e = timed(NANOKV_K_LOW, 2, bst, [&] {
          cudaError_t e2 = simt_low_prep(q, Tq, ck, qred, qc, bst);
          if (e2 == cudaSuccess) e2 = simt_attend_low(qred, qc, Tq, ck, cv, lk_, lv_, 0, r.T_l, softmax_scale, p, bst);
          return e2;
        });
      }
    }
    if (e == cudaSuccess && r.nred) {
      // reduced heads: reduce their queries once, then one launch per width;
      // beside the other classes, on helper streams 3 (the reduction, the
      // 32- and 96-wide launches) and 4 (the 64-wide launch, after the
      // reduction)
      void *qr = ws + r.off_qred;
      cudaStream_t rs[2] = {bst, bst};
      if (bs) {
        rs[0] = bstream(3);
        if (e == cudaSuccess) rs[1] = bstream(4);
        if (e != cudaSuccess) return cuda_status(e, "routed fork");
      }
      e = timed(NANOKV_K_LOW, 1, rs[0], [&] {
        return reduce_queries(q, Tq, ck.H, lowdim->U, HeadSel{lists + (size_t)HC_COUNT * ck.H, r.nred}, r.dims, qr,
                              rs[0]);
      });
      if (bs && e == cudaSuccess) {
        e = cudaEventRecord(bs->aux, rs[0]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(rs[1], bs->aux, 0);
      }
      const LowdimTables tb = lowdim_tables(ck, cv, lowdim->aux);
      Codec ckr = ck, cvr = cv;
      ckr.D = tb.D[0];
      ckr.centers = tb.cen[0];
      cvr.D = tb.D[1];
      cvr.centers = tb.cen[1];
      ckr.aux = cvr.aux = nullptr;
      const int width[3] = {32, 64, 96};
      for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
        const int c = HC_R32 + i;
        if (!k.ncls[c]) continue;
        cudaStream_t cs_ = rs[i == 1 ? 1 : 0];
        e = timed(NANOKV_K_LOW, 1, cs_, [&] {
          return tc_attend_reduced(width[i], qr, Tq, ckr, cvr, lowdim->W, lk_, lv_, 0, r.T_l, softmax_scale, p, cs_,
                                   sel(c));
        });
      }
      if (bs && e == cudaSuccess) e = join(3);
      if (bs && e == cudaSuccess) e = join(4);
    }
    if (e == cudaSuccess) e = join(0);
    if (e != cudaSuccess) return cuda_status(e, "routed low-set launch");
    pl.O[pl.n] = p.O;
    pl.LSE[pl.n++] = p.LSE;
  }
  if (on[1]) {
    Part p{(float *)(ws + w.off_O[1]), (float *)(ws + w.off_L[1])};
    cudaStream_t bst = bstream(1);
    if (e != cudaSuccess) return cuda_status(e, "routed fork");
    e = timed(NANOKV_K_FULL, 1, bst, [&] {
      return k.tc_full ? tc_attend_full(q, Tq, ck, cv, hs[0][0], hs[0][1], 0, r.T_f, softmax_scale, p, splits,
                                        w.osz / sizeof(float), w.lsz / sizeof(float), bst, false)
                       : simt_attend_full(q, Tq, ck, cv, hs[0][0], hs[0][1], 0, r.T_f, softmax_scale, p, bst);
    });
    if (e == cudaSuccess) e = join(1);
    if (e != cudaSuccess) return cuda_status(e, "routed full-set launch");
    for (int z = 0; z < w.nparts[1]; ++z) {
      pl.O[pl.n] = (const float *)(ws + w.off_O[1] + z * w.osz);
      pl.LSE[pl.n++] = (const float *)(ws + w.off_L[1] + z * w.lsz);
    }
  }
  if (on[2]) {
    Part p{(float *)(ws + w.off_O[2]), (float *)(ws + w.off_L[2])};
    cudaStream_t bst = bstream(2);
    if (e != cudaSuccess) return cuda_status(e, "routed fork");
    e = timed(NANOKV_K_DENSE, 1, bst, [&] {
      return k.tc_dense ? tc_attend_dense(q, Tq, ck.H, ck.d, k_cur, v_cur, T_cur, softmax_scale, p, bst, false)
                        : simt_attend_dense(ck.prec, q, Tq, ck.H, ck.d, k_cur, v_cur, T_cur, softmax_scale, p, bst);
    });
    if (e == cudaSuccess) e = join(2);
    if (e != cudaSuccess) return cuda_status(e, "routed current-chunk launch");
    pl.O[pl.n] = p.O;
    pl.LSE[pl.n++] = p.LSE;
  }
  if (lk.owns_lock()) lk.unlock();
  e = timed(NANOKV_K_MERGE, 1, st,
            [&] { return lse_merge_launch(pl, Tq, ck.H, ck.d, out, ck.prec, lse_out, st); });
  return cuda_status(e, "routed merge launch");
}

size_t nanokv_lowdim_aux_bytes(const nanokv_codec *ck_, const nanokv_codec *cv_) {
  Codec ck, cv;
  if (check_codec(ck_, "lowdim ck", false, &ck) || check_codec(cv_, "lowdim cv", false, &cv)) return 0;
  return lowdim_codecs_ok(ck, cv) ? lowdim_aux_bytes(ck, cv) : 0;
}

int nanokv_lowdim_prepare(const nanokv_codec *ck_, const nanokv_codec *cv_, const nanokv_lowdim *ld, void *stream) {
  ApiRange range("nanokv_lowdim_prepare");
  Codec ck, cv;
  int s;
  if ((s = check_codec(ck_, "lowdim ck", false, &ck))) return s;
  if ((s = check_codec(cv_, "lowdim cv", false, &cv))) return s;
  if (!lowdim_codecs_ok(ck, cv))
    return fail(NANOKV_ERR_UNSUPPORTED, "lowdim: needs bf16 codecs with d = 128 and equal H and r for K and V");
  if (!ld || !ld->U || !ld->W || !ld->aux || !aligned16(ld->U) || !aligned16(ld->W) || !aligned16(ld->aux))
    return fail(NANOKV_ERR_INVALID, "lowdim: U, W and aux must be non-NULL and 16-byte aligned");
  return cuda_status(lowdim_prepare(ck, cv, ld->U, ld->W, ld->aux, (cudaStream_t)stream), "lowdim prepare launch");
}

int nanokv_lowdim_analytic(const nanokv_codec *c_, void *maps, void *stream) {
  ApiRange range("nanokv_lowdim_analytic");
  Codec c;
  int s;
  if ((s = check_codec(c_, "lowdim analytic", false, &c))) return s;
  if (c.prec != PREC_BF16 || c.d != 128)
    return fail(NANOKV_ERR_UNSUPPORTED, "lowdim analytic: needs a bf16 codec with d = 128");
  if (!maps || !aligned16(maps)) return fail(NANOKV_ERR_INVALID, "lowdim analytic: maps NULL or misaligned");
  return cuda_status(lowdim_analytic(c, maps, (cudaStream_t)stream), "lowdim analytic launch");
}

size_t nanokv_calibrate_workspace(int64_t N, int32_t J, int32_t C) {
  if (N < 1 || J < 32 || J > 3072 || (J & 31) || C < 1 || C > 256) return 0;
  return calibrate_workspace(N, J, C);
}

int nanokv_calibrate(const void *x, int32_t dtype, int64_t N, int32_t J, int32_t C, int32_t r,
                     const float *init_centers, int32_t rounds, void *centers_out, void *D_out, void *E_out,
                     uint8_t *ids_out, float *eigenvalues_out, void *workspace, size_t workspace_bytes,
                     void *stream) {
  ApiRange range("nanokv_calibrate");
  const int prec = io_prec(dtype);
  if (prec < 0) return fail(NANOKV_ERR_UNSUPPORTED, "calibrate: dtype must be F32 or BF16");
  if (N < 1 || J < 32 || J > 3072 || (J & 31))
    return fail(NANOKV_ERR_INVALID, "calibrate: N=%lld must be >= 1 and J=%d a multiple of 32 in [32, 3072]",
                (long long)N, J);
  if (C < 1 || C > 256 || r < 1 || r > J || rounds < 0 || rounds > 1000)
    return fail(NANOKV_ERR_INVALID, "calibrate: C=%d (1..256), r=%d (1..J), rounds=%d (0..1000)", C, r, rounds);
  if (!x || !init_centers || !centers_out || !D_out || !E_out || !workspace)
    return fail(NANOKV_ERR_INVALID, "calibrate: NULL pointer");
  if (!aligned16(x) || !aligned16(init_centers) || !aligned16(workspace))
    return fail(NANOKV_ERR_INVALID, "calibrate: x, init_centers and workspace must be 16-byte aligned");
  const size_t need = calibrate_workspace(N, J, C);
  if (workspace_bytes < need)
    return fail(NANOKV_ERR_INVALID, "calibrate: workspace needs %zu bytes, got %zu", need, workspace_bytes);
  CalibArgs a{};
  a.x = x;
  a.N = N;
  a.J = J;
  a.C = C;
  a.r = r;
  a.rounds = rounds;
  a.prec = prec;
  a.init = init_centers;
  a.centers = centers_out;
  a.D = D_out;
  a.E = E_out;
  a.ids = ids_out;
  a.evals = eigenvalues_out;
  calibrate_carve(a, workspace);
  return cuda_status(calibrate_launch(a, (cudaStream_t)stream), "calibrate");
}

int nanokv_lse_merge(int32_t n, const float *const *o_parts, const float *const *lse_parts,
                     int64_t Tq, int32_t H, int32_t d, void *out, int32_t out_dtype,
                     float *lse_out, void *stream) {
  ApiRange range("nanokv_lse_merge");
  if (n < 1 || n > kMaxParts) return fail(NANOKV_ERR_INVALID, "merge: n=%d out of range [1,%d]", n, kMaxParts);
  if (Tq < 0 || H < 1 || d < 4 || (d & 3)) return fail(NANOKV_ERR_INVALID, "merge: bad sizes (d must be a multiple of 4)");
  const int op = io_prec(out_dtype);
  if (op < 0) return fail(NANOKV_ERR_UNSUPPORTED, "merge: out_dtype must be F32 or BF16");
  if (Tq == 0) return NANOKV_OK;
  if (!o_parts || !lse_parts || !out) return fail(NANOKV_ERR_INVALID, "merge: NULL pointer");
  PartList pl{};
  for (int b = 0; b < n; ++b) {
    if (!o_parts[b] || !lse_parts[b]) return fail(NANOKV_ERR_INVALID, "merge: NULL part %d", b);
    if (!aligned16(o_parts[b])) return fail(NANOKV_ERR_INVALID, "merge: part %d misaligned", b);
    pl.O[b] = o_parts[b];
    pl.LSE[b] = lse_parts[b];
  }
  pl.n = n;
  if (!aligned16(out)) return fail(NANOKV_ERR_INVALID, "merge: out misaligned");
  cudaStream_t st = (cudaStream_t)stream;
  return cuda_status(
      timed(NANOKV_K_MERGE, 1, st, [&] { return lse_merge_launch(pl, Tq, H, d, out, op, lse_out, st); }),
      "merge launch");
}

int nanokv_timing_enable(int32_t on) {
  return g_timing.exchange(on ? 1 : 0);
}

int nanokv_timing_read(double *ms_total, int64_t *launches) {
  std::vector<TimingRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_tmu);
    recs.swap(g_recs);
  }
  double tot[NANOKV_K_COUNT] = {0};
  int status = NANOKV_OK;
  for (auto &r : recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess && status == NANOKV_OK) status = cuda_status(e, "timing read");
    tot[r.kid] += ms;
  }
  {
    std::lock_guard<std::mutex> lk(g_tmu);
    for (auto &r : recs) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
  }
  for (int k = 0; k < NANOKV_K_COUNT; ++k) {
    if (ms_total) ms_total[k] = tot[k];
    const int64_t n = g_launches[k].exchange(0);
    if (launches) launches[k] = n;
  }
  return status;
}

}  // extern "C"
