// nanokv_attend_static: nanokv_attend for callers that cannot allocate device
// memory.  Its scratch (the fp32 per-branch partial outputs and, on the
// CUDA-core low-dim path, the reduced-query buffers) lives in one fixed device
// array compiled into this library instead of a caller-provided workspace.
#include "../../include/nanokv.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace nanokv {
int set_error(int status, const char *msg);  // api.cu
}

namespace {

// Upper bound on the scratch one call may use.  Every GPU that loads the
// library keeps this much device memory until the process exits.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB

__device__ __align__(256) unsigned char g_attend_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// the current driver context, through the runtime's entry-point query (the
// library takes no link-time dependency on the driver library)
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext *);
  static Fn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? (Fn)p
               : (Fn) nullptr;
  }();
  CUcontext c = nullptr;
  if (fn) fn(&c);
  return c;
}

// Device address of the scratch array on the current device.  Host code can
// only name the array's host-side stand-in, so the address is looked up (with
// that device current) and cached per device together with the context it
// belongs to: after a device reset, or under another context of the same
// device, the array lives at a new address and is looked up again.
int scratch_for_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nanokv::set_error(NANOKV_ERR_CUDA, "attend_static: no usable current device");
  CUcontext ctx = current_context();  // NULL before the runtime has made the primary context current
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attend_scratch);
    if (e != cudaSuccess || !p)
      return nanokv::set_error(NANOKV_ERR_CUDA, "attend_static: cudaGetSymbolAddress of the scratch array failed");
    if (!ctx) ctx = current_context();  // the lookup made the primary context current
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return NANOKV_OK;
}

}  // namespace

extern "C" int nanokv_attend_static(const void *q, int32_t io_dtype, int64_t Tq, const nanokv_codec *ck,
                                    const nanokv_codec *cv, const nanokv_hist *hk, const nanokv_hist *hv,
                                    int64_t T, int64_t T_full, const void *k_cur, const void *v_cur,
                                    int64_t T_cur, float softmax_scale, void *out, float *lse_out,
                                    void *stream) {
  // sizes beyond the array are refused before anything touches the GPU; an
  // invalid argument yields 0 here and is reported by nanokv_attend below
  const size_t need = nanokv_attend_workspace(Tq, ck, cv, T, T_full, T_cur);
  if (need > kStaticScratchBytes)
    return nanokv::set_error(NANOKV_ERR_INVALID,
                             "attend_static: this call needs more scratch than the library's fixed 32 MiB "
                             "array; use nanokv_attend with a caller-provided workspace");
  void *scratch = nullptr;
  const int s = scratch_for_current_device(&scratch);
  if (s != NANOKV_OK) return s;
  return nanokv_attend(q, io_dtype, Tq, ck, cv, hk, hv, T, T_full, k_cur, v_cur, T_cur, softmax_scale, out,
                       lse_out, scratch, kStaticScratchBytes, stream);
}
