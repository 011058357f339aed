// Windowed no-repeat n-gram ban
// ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.3): inside the
// history window, every token that would complete an n-gram already present
// there gets logit -inf.
//
// One warp per row.  The row's history (at most `window` int32, 512 bytes at
// the pages' window of 128) is read through the read-only cache; lane i tests
// candidate starts i, i+32, ...  Each candidate compares its (n-1)-gram with
// the row's (n-1)-suffix and, on a match, stores -inf over the follower's
// logit.  Only banned columns are written: the kernel moves ~0.5 KB per row
// plus one 4-byte store per ban, so it is bound by launch latency, not HBM.
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace rswa {
namespace {

constexpr int kWarpsPerBlock = 4;

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    ngram_mask_kernel(float *__restrict__ logits, int64_t ld, const int32_t *__restrict__ history,
                      int64_t hist_ld, const int32_t *__restrict__ hist_len, int rows, int vocab,
                      int n, int window, int *err) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  // programmatic dependent launch: the previous kernel (which may have written
  // the logits or the history) has completed past this point; the next launch
  // may start scheduling meanwhile
  grid_dependency_wait();
  allow_dependents();
  if (row >= rows) return;
  const int32_t *hist = history + (int64_t)row * hist_ld;
  const int h = hist_len ? __ldg(hist_len + row) : window;
  if (h < 0 || h > window) {
    if (lane == 0 && err) atomicOr(err, RSWA_DEVERR_BAD_LENGTH);
    return;
  }
  bool bad = false;
  for (int i = lane; i < h; i += 32) {
    const int tok = __ldg(hist + i);
    bad |= tok < 0 || tok >= vocab;
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0 && err) atomicOr(err, RSWA_DEVERR_BAD_TOKEN);
    return;
  }
  if (h < n) return;
  const int m = n - 1;             // prefix length
  const int32_t *suffix = hist + (h - m);
  float *lrow = logits + (int64_t)row * ld;
  for (int i = lane; i + n <= h; i += 32) {
    bool match = true;
    for (int j = 0; j < m; ++j) {
      if (__ldg(hist + i + j) != __ldg(suffix + j)) {
        match = false;
        break;
      }
    }
    if (match) lrow[__ldg(hist + i + m)] = -INFINITY;
  }
}

}  // namespace

cudaError_t launch_ngram(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                         const int32_t *hist_len, int rows, int vocab, int n, int window,
                         int *err, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const int blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)blocks);
  lc.blockDim = dim3(kWarpsPerBlock * 32);
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, ngram_mask_kernel, logits, ld, history, hist_ld, hist_len, rows,
                            vocab, n, window, err);
}

}  // namespace rswa
