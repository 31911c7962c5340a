// Gather of routed history tokens (NanoKV-Fast, Table 7: full-dimensional
// routing by token ranges and by head).  A routing policy splits the history
// into the tokens read full-dim and the rest, read low-dim; each set is
// copied into a contiguous compressed history (ids, packed codes, scales of
// both branches), so that the attention kernels read it as one range.
// Attention does not depend on the order of its keys, so the gathered sets
// give the same result as reading the tokens in place.
#include "common.cuh"

namespace nanokv {

namespace {

__global__ void __launch_bounds__(256) gather_kernel(GatherSegs full, GatherSegs low, GatherArgs A) {
  // head lists: the heads of each class, in order
  if (A.head_lists && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    int n[HC_COUNT] = {}, nr = 0;
    for (int h = 0; h < A.H; ++h) {
      const int c = A.head_class[h] < HC_COUNT ? A.head_class[h] : HC_LOW;
      A.head_lists[c * A.H + n[c]++] = h;
      if (c >= HC_R32) A.head_lists[HC_COUNT * A.H + nr++] = h;  // and every reduced head
    }
  }
  const int set = blockIdx.y;
  const GatherSegs &sg = set ? low : full;
  const int64_t n = A.n_out[set];
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
    // the segment holding output position p: the last one starting at or before it
    int lo = 0, hi = sg.n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sg.dst[mid] <= p) lo = mid;
      else hi = mid - 1;
    }
    const int64_t s = sg.src[lo] + (p - sg.dst[lo]);
#pragma unroll
    for (int br = 0; br < 2; ++br) {
      A.d_ids[set][br][p] = A.ids[br][s];
      const int sb = A.scale_bytes;
      for (int b = 0; b < sb; ++b) A.d_scales[set][br][p * sb + b] = A.scales[br][s * sb + b];
      const int rb = A.row_bytes[br];
      const uint8_t *src = A.codes[br] + s * rb;
      uint8_t *dst = A.d_codes[set][br] + p * rb;
      if ((rb & 15) == 0) {
        for (int b = 0; b < rb; b += 16)
          *reinterpret_cast<uint4 *>(dst + b) = *reinterpret_cast<const uint4 *>(src + b);
      } else {
        for (int b = 0; b < rb; ++b) dst[b] = src[b];
      }
    }
  }
}

}  // namespace

cudaError_t gather_launch(const GatherSegs &full, const GatherSegs &low, const GatherArgs &a, cudaStream_t st) {
  const int64_t n = a.n_out[0] > a.n_out[1] ? a.n_out[0] : a.n_out[1];
  int64_t blocks = (n + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 2048) blocks = 2048;
  gather_kernel<<<dim3((unsigned)blocks, 2), 256, 0, st>>>(full, low, a);
  return cudaGetLastError();
}

}  // namespace nanokv
