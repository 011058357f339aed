// Fused windowed n-gram ban + top-k selection over the vocabulary (greedy
// decoding at k = 1, optional sampling among the k survivors).
//
// Method ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.3): inside
// the sliding window of the generated history, every token that would repeat
// an n-gram of size ngram_size gets score -inf; the next token is then chosen
// from the masked scores.  Selection follows a total order: larger masked
// value first, the lower column first among equal values; NaN ranks as -inf.
//
// Design (HBM-bound: each logit is read once from DRAM):
//  - One thread-block cluster of C = ceil(vocab / 16384) CTAs per row; each
//    CTA streams its 16,384 columns (64 per thread, in four batches of four
//    16-byte loads, two batches in flight) and keeps, per thread, the first
//    two maxima of its columns in increasing column order.
//  - The ban: the row's history is copied to shared memory asynchronously at
//    kernel start and worked out while the last batches are in flight; every
//    thread tests candidate starts of the windowed n-gram match; the banned
//    tokens in this CTA's columns go into a shared-memory bitmap (and, on
//    request, -inf is stored over them in the logits).  A thread whose best
//    column is banned falls back on its second, and rescans its columns
//    (from L2) only if both are banned.
//  - Every column gets a 64-bit key: the order-preserving image of its masked
//    value in the high word, (2^32 - 1 - column) in the low word, so keys
//    are distinct and "larger key" is exactly the selection order.
//  - k = 1 (its own kernel): the thread maxima are reduced over the warp, the
//    CTA and, through distributed shared memory, the cluster's leader.  The
//    CTA's column range is requested into L2 by bulk prefetches at kernel
//    start, so the row leaves DRAM at full depth.
//  - k > 1: the leader gathers the C x 256 thread maxima and finds their k-th
//    largest, T, by a CTA-local radix select (8 bits per pass, over the keys'
//    offsets from the smallest of them).  At least k
//    keys of the row are >= T, and they all lie in the k threads whose
//    maximum is >= T.  A thread whose second largest key is known and below T
//    sends only its maximum; the others with a maximum >= T reread their
//    columns (from L2) and send every key >= T.  The leader ranks up to 256
//    candidates directly (each thread counts the larger ones), else first
//    radix-selects the k-th largest among them.
//  - Sampling: p_i proportional to exp((x_i - x_0) / T) over the k survivors
//    (x_0 the largest), inverse CDF at the caller's uniform u in [0, 1).
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace rswa {
namespace {

constexpr int kThreads = 256;
constexpr int kF4PerThread = 16;
constexpr int kEPT = 4 * kF4PerThread;     // columns per thread
constexpr int kChunk = kThreads * kEPT;    // columns per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTopkCluster = 16;        // vocab <= 16 * kChunk
// leader's candidate buffer: the C x 256 thread maxima first, then the keys
// >= T (at most 64 per thread of the k threads whose maximum is >= T)
constexpr int kTopkCandidates = 64 * kTopkMax;
static_assert(kMaxTopkCluster * kThreads <= kTopkCandidates, "thread maxima fit the buffer");
static_assert(kTopkMax <= kThreads, "one thread per selected key");


// Inverse of the order image (for the reported values).
__device__ __forceinline__ float ord_value(uint32_t o) {
  const uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  return __uint_as_float(u);
}

// Order-preserving image of a masked value, branch-free: NaN -> -inf via
// fmaxf, -0 -> +0 via the addition, then the sign-dependent flip.
__device__ __forceinline__ uint32_t ord_fast(float x) {
  const float y = fmaxf(x, -INFINITY) + 0.0f;
  const uint32_t u = __float_as_uint(y);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

struct TopkArgs {
  float *logits;
  int64_t ld;
  const int32_t *history;
  int64_t hist_ld;
  const int32_t *hist_len;
  int rows, vocab, n, window, k, mask_in_place;
  const float *uniform;
  float inv_temp_log2e;  // log2(e) / T
  int32_t *top_idx;
  float *top_val;
  int32_t *token;
  int *err;
};

// Completes the staged history (hist_s, `window` ints), checks it, and marks the banned tokens that fall in [col0, col0 + kChunk)
// in ban_bits (zeroed here), storing -inf over them when asked.  Returns the
// row's error bits (the same in every CTA of the row).  Ends with a barrier.
// Starts the copy of row `row`'s history (the first `window` tokens) into
// shared memory; ban_prologue completes it.
__device__ __forceinline__ void stage_history(const TopkArgs &a, int row, int32_t *hist_s) {
  const int32_t *hist = a.history + (int64_t)row * a.hist_ld;
  for (int i = threadIdx.x; i < a.window; i += kThreads) cp_async_4(hist_s + i, hist + i);
}

__device__ int ban_prologue(const TopkArgs &a, int row, int col0, uint32_t *ban_bits,
                            int32_t *hist_s) {
  const int tid = threadIdx.x;
  const int h = a.hist_len ? __ldg(a.hist_len + row) : a.window;
  const bool len_bad = h < 0 || h > a.window;
  for (int i = tid; i < kChunk / 32; i += kThreads) ban_bits[i] = 0;
  cp_async_wait_all();
  __syncthreads();
  bool tok_bad = false;
  if (!len_bad)
    for (int i = tid; i < h; i += kThreads) {
      const int tok = hist_s[i];
      tok_bad |= tok < 0 || tok >= a.vocab;
    }
  const int any_bad = __syncthreads_or(tok_bad);
  if (len_bad) return RSWA_DEVERR_BAD_LENGTH;
  if (any_bad) return RSWA_DEVERR_BAD_TOKEN;
  if (h >= a.n) {
    const int m = a.n - 1;
    const int32_t *suffix = hist_s + (h - m);
    float *lrow = a.logits + (int64_t)row * a.ld;
    for (int i = tid; i + a.n <= h; i += kThreads) {
      int j = 0;
      while (j < m && hist_s[i + j] == suffix[j]) ++j;
      if (j < m) continue;
      const int f = hist_s[i + m] - col0;
      if (f >= 0 && f < kChunk) {
        atomicOr(&ban_bits[f >> 5], 1u << (f & 31));
        if (a.mask_in_place) lrow[col0 + f] = -INFINITY;
      }
    }
  }
  __syncthreads();
  return 0;
}

// Outputs of a rejected row (written by the leader CTA only).
__device__ void reject_row(const TopkArgs &a, int row, int rank) {
  if (rank != 0) return;
  for (int i = threadIdx.x; i < a.k; i += kThreads) {
    a.top_idx[(int64_t)row * a.k + i] = -1;
    if (a.top_val) a.top_val[(int64_t)row * a.k + i] = __int_as_float(0x7fc00000);
  }
  if (threadIdx.x == 0 && a.token) a.token[row] = -1;
}

// The streaming pass shared by both kernels: each thread reads its 64 columns
// once (two batches of four 16-byte loads in flight; in the top-1 form the
// CTA's whole range is first requested into L2 by bulk prefetches, so the
// row streams from DRAM at full depth) and keeps the two first
// maxima of them in increasing column order; the ban is worked out while the
// last two batches are in flight (top-1 form) or right after the stream
// (top-k form); the history was copied asynchronously at the start.  If a thread's best is banned its second is the answer, unless
// that is banned too, in which case the thread rescans its columns (from L2)
// skipping banned ones -- which needs two banned tokens among one thread's 64
// columns.  Returns the thread's largest masked key ((order image of the
// masked value) << 32 | ~column), 0 if it has no column, and sets *bad to
// the row's error bits (the same in every CTA of the row).  With `second`,
// also its second largest masked key where the two tracked maxima give it
// exactly (neither banned, the second finite), else kKeyUnknown.
constexpr unsigned long long kKeyUnknown = ~0ull;  // above every real key
template <bool kEvictFirst>
__device__ __forceinline__ unsigned long long stream_thread_max(const TopkArgs &a, int row,
                                                                int col0, uint32_t *ban_bits,
                                                                int32_t *hist_s, int *bad,
                                                                unsigned long long *second = nullptr) {
  const int tid = threadIdx.x;
  const float *lrow = a.logits + (int64_t)row * a.ld;
  if (kEvictFirst) {
    // single-pass (top-1) form: the CTA's whole column range on its way into
    // L2 at once (the loads below keep only two batches per thread in
    // flight).  The row and col0 are 16-byte aligned, and col0 < vocab.
    // (The two-pass top-k form measured slower with it.)
    const int ncols = min(kChunk, a.vocab - col0);
    const uint32_t bytes = (uint32_t)(ncols * 4) & ~15u;
    constexpr uint32_t kPiece = 4096;
    for (uint32_t off = (uint32_t)tid * kPiece; off < bytes; off += kThreads * kPiece)
      bulk_prefetch_l2(reinterpret_cast<const char *>(lrow + col0) + off,
                       bytes - off < kPiece ? bytes - off : kPiece);
  }
  stage_history(a, row, hist_s);
  constexpr int kBatch = 4;
  static_assert(kF4PerThread == 4 * kBatch, "four batches per thread");
  auto load_batch = [&](float4 *dst, int i0) {
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int c = col0 + 4 * (tid + kThreads * (i0 + i));
      dst[i] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      // volatile: issued here, in this order, not sunk to the first use
      if (c < a.vocab) {
        if (kEvictFirst)
          asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(dst[i].x), "=f"(dst[i].y), "=f"(dst[i].z), "=f"(dst[i].w)
                       : "l"(lrow + c));
        else
          asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(dst[i].x), "=f"(dst[i].y), "=f"(dst[i].z), "=f"(dst[i].w)
                       : "l"(lrow + c));
      }
    }
  };
  // columns in increasing order: strict comparisons keep the first of equals
  const int first_col = col0 + 4 * tid;
  float b1 = -INFINITY, b2 = -INFINITY;
  int i1 = first_col, i2 = first_col;
  auto consume = [&](const float4 *x, int i0) {
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int c = col0 + 4 * (tid + kThreads * (i0 + i));
      const float e[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float v = c + u < a.vocab ? e[u] : -INFINITY;
        const bool gt1 = v > b1, gt2 = v > b2;
        b2 = gt1 ? b1 : (gt2 ? v : b2);
        i2 = gt1 ? i1 : (gt2 ? c + u : i2);
        b1 = gt1 ? v : b1;
        i1 = gt1 ? c + u : i1;
      }
    }
  };
  float4 x0[kBatch], x1[kBatch];
  load_batch(x0, 0);
  load_batch(x1, kBatch);
  consume(x0, 0);
  load_batch(x0, 2 * kBatch);
  consume(x1, kBatch);
  load_batch(x1, 3 * kBatch);
  // The ban's barriers hold every warp of the CTA.  The top-1 form works it
  // out while its last two batches are in flight (10.7 against 11.2 us per
  // call with it after the stream); the top-k form, which has a second pass
  // behind it, after the stream (20.45 against 20.7 us).
  if (kEvictFirst) {
    *bad = ban_prologue(a, row, col0, ban_bits, hist_s);
    if (*bad) return 0;
  }
  consume(x0, 2 * kBatch);
  consume(x1, 3 * kBatch);
  if (!kEvictFirst) {
    *bad = ban_prologue(a, row, col0, ban_bits, hist_s);
    if (*bad) return 0;
  }

  const auto banned = [&](int col) {
    const int f = col - col0;
    return ((ban_bits[f >> 5] >> (f & 31)) & 1u) != 0;
  };
  if (second)
    *second = (b1 != -INFINITY && !banned(i1) && b2 != -INFINITY && !banned(i2) && i2 < a.vocab)
                  ? ((unsigned long long)ord_fast(b2) << 32) | (0xFFFFFFFFu - (uint32_t)i2)
                  : kKeyUnknown;
  float best = b1;
  int bi = i1;
  if (b1 != -INFINITY && banned(i1)) {
    if (b2 == -INFINITY) {
      best = -INFINITY;  // everything left ranks as -inf: the lowest column
      bi = first_col;
    } else if (!banned(i2)) {
      best = b2;
      bi = i2;
    } else {
      // rescan with the ban applied, 8 loads in flight at a time
      best = -INFINITY;
      bi = first_col;
      for (int h0 = 0; h0 < kF4PerThread; h0 += 2 * kBatch) {
        float4 y[2 * kBatch];
#pragma unroll
        for (int i = 0; i < 2 * kBatch; ++i) {
          const int c = col0 + 4 * (tid + kThreads * (h0 + i));
          y[i] = c < a.vocab ? *reinterpret_cast<const float4 *>(lrow + c)
                             : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 2 * kBatch; ++i) {
          const int c = col0 + 4 * (tid + kThreads * (h0 + i));
          const float e[4] = {y[i].x, y[i].y, y[i].z, y[i].w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (c + u < a.vocab && e[u] > best && !banned(c + u)) {
              best = e[u];
              bi = c + u;
            }
        }
      }
    }
  }
  return bi < a.vocab ? ((unsigned long long)ord_fast(best) << 32) | (0xFFFFFFFFu - (uint32_t)bi)
                      : 0ull;
}

// k = 1: the largest masked key of the row, nothing held.
__global__ void __launch_bounds__(kThreads, 4)  // 4 CTAs/SM: 64 rows x 8 CTAs in one wave
    ngram_top1_kernel(const TopkArgs a) {
  __shared__ uint32_t ban_bits[kChunk / 32];
  __shared__ unsigned long long warp_best[kWarps];
  __shared__ unsigned long long cta_best[kMaxTopkCluster];
  extern __shared__ int32_t hist_s[];
  const int C = (int)(gridDim.x / (unsigned)a.rows);
  const int row = (int)(blockIdx.x / (unsigned)C);
  const int rank = (int)(blockIdx.x % (unsigned)C);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col0 = rank * kChunk;
  // programmatic dependent launch: the previous kernel (which may have written
  // the logits or the history) has completed past this point, and the next
  // launch may start scheduling its CTAs while this one runs
  grid_dependency_wait();
  allow_dependents();
  // arrive now, wait before the first remote store: no CTA then writes into a
  // peer that has not started, and the wait costs nothing by that time
  cluster_arrive_relaxed();
  int bad = 0;
  unsigned long long key = stream_thread_max<true>(a, row, col0, ban_bits, hist_s, &bad);
  if (bad) {  // the same in every CTA of the row
    if (rank == 0 && tid == 0 && a.err) atomicOr(a.err, bad);
    reject_row(a, row, rank);
    cluster_wait_acquire();  // leave the start-of-kernel phase balanced
    return;
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, off));
  if (lane == 0) warp_best[warp] = key;
  __syncthreads();
  cluster_wait_acquire();  // every CTA of the cluster has started
  if (tid == 0) {
    unsigned long long b = 0;
    for (int i = 0; i < kWarps; ++i) b = max(b, warp_best[i]);
    st_cluster_u64(map_to_rank(&cta_best[rank], 0), b);  // into the leader
  }
  __syncwarp();
  cluster_arrive_release();
  cluster_wait_acquire();
  if (rank == 0 && tid == 0) {
    unsigned long long b = 0;
    for (int r = 0; r < C; ++r) b = max(b, cta_best[r]);
    const int col = (int)(0xFFFFFFFFu - (uint32_t)b);
    a.top_idx[row] = col;
    if (a.top_val) a.top_val[row] = ord_value((uint32_t)(b >> 32));
    if (a.token) a.token[row] = col;
  }
}

// Threshold T with exactly k of the n keys (which may repeat) at or above it
// when the k-th largest key is unique among them, and at least k otherwise:
// a radix select over d = key - (smallest key), from the top bit of the
// largest d down, 8 bits per pass, stopping when the chosen digit's bin holds
// exactly the keys still needed.  Taking digits of d rather than of the key
// spreads keys that share their leading bits (thread maxima of N(0, 1)
// logits mostly share sign and exponent) over the bins from the first pass,
// so the histogram atomics rarely collide.  CTA-wide; keys in shared memory;
// ends with a barrier.
// (smallest, largest) of the keys: span[i] and span[kSpanHalf + i] for
// i < nspan hold partial minima and maxima already (nspan > 0), or the CTA
// works them out here (nspan = 0).
constexpr int kSpanHalf = kMaxTopkCluster > kWarps ? kMaxTopkCluster : kWarps;
__device__ unsigned long long cta_kth_threshold(const unsigned long long *keys, int n, int k,
                                                uint32_t *hist, uint32_t *scan, uint32_t *sel,
                                                unsigned long long *span, int nspan) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (nspan == 0) {
    unsigned long long lo = ~0ull, hi = 0;
    for (int i = tid; i < n; i += kThreads) {
      lo = min(lo, keys[i]);
      hi = max(hi, keys[i]);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
      span[warp] = lo;
      span[kSpanHalf + warp] = hi;
    }
    nspan = kWarps;
    __syncthreads();
  }
  unsigned long long lo = span[0], hi = span[kSpanHalf];
  for (int i = 1; i < nspan; ++i) {
    lo = min(lo, span[i]);
    hi = max(hi, span[kSpanHalf + i]);
  }
  if (lo == hi) {
    __syncthreads();  // span is rewritten by the next call
    return lo;
  }
  // bits [lo_shift, hi_shift) of d form this pass's digit; the bits above
  // are `prefix` for every key still in the running
  int hi_shift = 64 - __clzll((long long)(hi - lo));
  int lo_shift = hi_shift > 8 ? hi_shift - 8 : 0;
  unsigned long long prefix = 0;
  uint32_t need = (uint32_t)k;
  for (;;) {
    hist[tid] = 0;
    __syncthreads();
    const uint32_t mask = (1u << (hi_shift - lo_shift)) - 1u;
    for (int i = tid; i < n; i += kThreads) {
      const unsigned long long d = keys[i] - lo;
      if (hi_shift >= 64 || (d >> hi_shift) == prefix)
        atomicAdd(&hist[(uint32_t)(d >> lo_shift) & mask], 1u);
    }
    __syncthreads();
    // bin (255 - tid); suffix sums = prefix scan of the reversed bins
    const int bin = 255 - tid;
    const uint32_t cnt = hist[bin];
    uint32_t inc = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += y;
    }
    if (lane == 31) scan[warp] = inc;
    __syncthreads();
    uint32_t before = 0;
    for (int i = 0; i < warp; ++i) before += scan[i];
    const uint32_t incl = before + inc;  // keys in bins >= bin
    if (incl >= need && incl - cnt < need) {
      sel[0] = (uint32_t)bin;
      sel[1] = need - (incl - cnt);
      sel[2] = cnt == need - (incl - cnt);
    }
    __syncthreads();
    prefix = (prefix << (hi_shift - lo_shift)) | sel[0];
    need = sel[1];
    const bool done = sel[2] || lo_shift == 0;
    hi_shift = lo_shift;
    lo_shift = lo_shift > 8 ? lo_shift - 8 : 0;
    __syncthreads();  // sel and hist are rewritten by the next pass
    if (done) break;
  }
  return lo + (prefix << hi_shift);
}

// k > 1, one cluster per row:
//  1. the streaming pass gives each thread its largest masked key;
//  2. the leader gathers the C x 256 thread maxima and finds the k-th largest,
//     T: at least k keys of the row are >= T, and any key >= T lies in one of
//     the k threads whose maximum is >= T, so at most 64 k keys are;
//  3. every CTA rereads its columns (from L2) and sends its keys >= T to the
//     leader;
//  4. the leader selects the k largest of those candidates exactly, orders
//     them, writes them and samples.
__global__ void __launch_bounds__(kThreads, 4)
    ngram_topk_kernel(const TopkArgs a) {
  __shared__ uint32_t ban_bits[kChunk / 32];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t scan[kWarps];
  __shared__ uint32_t sel[3];
  __shared__ unsigned long long span[2 * kSpanHalf];  // leader: the CTAs' (min, max) thread maxima
  __shared__ unsigned long long wspan[2 * kWarps];
  __shared__ unsigned long long thr;               // T, written by the leader into every CTA
  __shared__ uint32_t n_cand, n_top;               // leader: candidates received, selected
  __shared__ unsigned long long sorted[kTopkMax];
  __shared__ unsigned long long top[kTopkMax];
  __shared__ float prob[kTopkMax];
  extern __shared__ __align__(16) uint8_t dyn[];
  unsigned long long *keybuf = reinterpret_cast<unsigned long long *>(dyn);  // kTopkCandidates
  int32_t *hist_s = reinterpret_cast<int32_t *>(dyn + kTopkCandidates * 8);
  const int C = (int)(gridDim.x / (unsigned)a.rows);
  const int row = (int)(blockIdx.x / (unsigned)C);
  const int rank = (int)(blockIdx.x % (unsigned)C);
  const int tid = threadIdx.x;
  const int col0 = rank * kChunk;
  const float *lrow = a.logits + (int64_t)row * a.ld;
  grid_dependency_wait();  // as in the greedy kernel
  allow_dependents();
  cluster_arrive_relaxed();
  if (tid == 0) {
    n_cand = 0;
    n_top = 0;
  }
  int bad = 0;
  unsigned long long key2;
  const unsigned long long key = stream_thread_max<false>(a, row, col0, ban_bits, hist_s, &bad,
                                                          &key2);
  if (bad) {  // the same in every CTA of the row
    if (rank == 0 && tid == 0 && a.err) atomicOr(a.err, bad);
    reject_row(a, row, rank);
    cluster_wait_acquire();
    return;
  }
  // ---- 2. thread maxima into the leader; T back to every CTA
  cluster_wait_acquire();  // every CTA of the cluster has started
  st_cluster_u64(map_to_rank(&keybuf[rank * kThreads + tid], 0), key);
  {
    // this CTA's smallest and largest thread maximum, for the leader's select
    unsigned long long mn = key, mx = key;
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if ((tid & 31) == 0) {
      wspan[tid >> 5] = mn;
      wspan[kWarps + (tid >> 5)] = mx;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < kWarps; ++w) {
        mn = min(mn, wspan[w]);
        mx = max(mx, wspan[kWarps + w]);
      }
      st_cluster_u64(map_to_rank(&span[rank], 0), mn);
      st_cluster_u64(map_to_rank(&span[kSpanHalf + rank], 0), mx);
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  if (rank == 0) {
    const unsigned long long T = cta_kth_threshold(keybuf, C * kThreads, a.k, hist, scan, sel, span, C);
    if (tid < C) st_cluster_u64(map_to_rank(&thr, tid), T);
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  // ---- 3. this CTA's keys >= T to the leader (its key buffer is free again).
  // A thread whose largest key is below T has none; one whose second largest
  // is known and below T has only its largest; any other thread with a key
  // >= T rereads its columns (from L2).
  {
    const unsigned long long T = thr;
    const uint32_t cand_addr = map_to_rank(keybuf, 0);
    const uint32_t count_addr = map_to_rank(&n_cand, 0);
    const bool only_first = key >= T && key2 < T;
    if (only_first) {
      const uint32_t slot = atom_add_cluster_u32(count_addr, 1u);
      if (slot < (uint32_t)kTopkCandidates) st_cluster_u64(cand_addr + 8u * slot, key);
    }
    const bool reread = key >= T && !only_first;
    for (int i0 = 0; reread && i0 < kF4PerThread; i0 += 8) {
      float4 y[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = col0 + 4 * (tid + kThreads * (i0 + i));
        y[i] = c < a.vocab ? *reinterpret_cast<const float4 *>(lrow + c)
                           : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = col0 + 4 * (tid + kThreads * (i0 + i));
        const uint32_t bits = ban_bits[(c - col0) >> 5] >> ((c - col0) & 31);
        const float e[4] = {y[i].x, y[i].y, y[i].z, y[i].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (c + u >= a.vocab) continue;
          const float vm = ((bits >> u) & 1u) ? -INFINITY : e[u];
          const unsigned long long kk =
              ((unsigned long long)ord_fast(vm) << 32) | (0xFFFFFFFFu - (uint32_t)(c + u));
          if (kk >= T) {
            const uint32_t slot = atom_add_cluster_u32(count_addr, 1u);
            if (slot < (uint32_t)kTopkCandidates) st_cluster_u64(cand_addr + 8u * slot, kk);
          }
        }
      }
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  if (rank != 0) return;  // the leader reads only its own shared memory from here

  // ---- 4. the k largest candidates, ordered.  Keys are distinct (they hold
  // the column).  Up to one candidate per thread: each counts the larger
  // ones, its rank, and the k first ranks are the answer in order.  More:
  // a radix select of the k-th largest, then the same ranking among those.
  const int k = a.k;
  const int nc = min((int)n_cand, kTopkCandidates);
  if (nc <= kThreads) {
    if (tid < nc) {
      const unsigned long long mine = keybuf[tid];
      int r = 0;
      for (int j = 0; j < nc; ++j) r += keybuf[j] > mine;
      if (r < k) sorted[r] = mine;
    }
    __syncthreads();
  } else {
    const unsigned long long T2 = cta_kth_threshold(keybuf, nc, k, hist, scan, sel, span, 0);
    for (int i = tid; i < nc; i += kThreads) {
      const unsigned long long kk = keybuf[i];
      if (kk >= T2) {
        const uint32_t slot = atomicAdd(&n_top, 1u);
        if (slot < (uint32_t)kTopkMax) top[slot] = kk;
      }
    }
    __syncthreads();
    if (tid < k) {
      const unsigned long long mine = top[tid];
      int r = 0;
      for (int j = 0; j < k; ++j) r += top[j] > mine;
      sorted[r] = mine;
    }
    __syncthreads();
  }
  if (tid < k) {
    const unsigned long long kk = sorted[tid];
    const int col = (int)(0xFFFFFFFFu - (uint32_t)kk);
    const float val = ord_value((uint32_t)(kk >> 32));
    a.top_idx[(int64_t)row * k + tid] = col;
    if (a.top_val) a.top_val[(int64_t)row * k + tid] = val;
    const float x0 = ord_value((uint32_t)(sorted[0] >> 32));
    prob[tid] = (val == -INFINITY || x0 == -INFINITY) ? 0.f : exp2f((val - x0) * a.inv_temp_log2e);
  }
  __syncthreads();
  if (tid < 32 && a.token) {
    // inverse CDF over the k (<= 64) survivors in rank order: warp 0 holds
    // survivors lane and lane + 32 and scans their probabilities; the draw is
    // the first survivor (p > 0) whose cumulative sum exceeds u * total, else
    // the last one with p > 0
    const int lane = tid;
    const float p_lo = lane < k ? prob[lane] : 0.f;
    const float p_hi = lane + 32 < k ? prob[lane + 32] : 0.f;
    float c_lo = p_lo, c_hi = p_hi;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y_lo = __shfl_up_sync(0xffffffffu, c_lo, off);
      const float y_hi = __shfl_up_sync(0xffffffffu, c_hi, off);
      if (lane >= off) {
        c_lo += y_lo;
        c_hi += y_hi;
      }
    }
    c_hi += __shfl_sync(0xffffffffu, c_lo, 31);
    const float total = __shfl_sync(0xffffffffu, c_hi, 31);
    int pick = 0;
    if (a.uniform && prob[0] > 0.f) {
      const float target = a.uniform[row] * total;
      const uint32_t over_lo = __ballot_sync(0xffffffffu, p_lo > 0.f && c_lo > target);
      const uint32_t over_hi = __ballot_sync(0xffffffffu, p_hi > 0.f && c_hi > target);
      const uint32_t pos_lo = __ballot_sync(0xffffffffu, p_lo > 0.f);
      const uint32_t pos_hi = __ballot_sync(0xffffffffu, p_hi > 0.f);
      if (over_lo) pick = __ffs(over_lo) - 1;
      else if (over_hi) pick = 32 + __ffs(over_hi) - 1;
      else pick = pos_hi ? 63 - __clz(pos_hi) : 31 - __clz(pos_lo);
    }
    if (lane == 0) a.token[row] = (int)(0xFFFFFFFFu - (uint32_t)sorted[pick]);
  }
}

}  // namespace

int topk_cluster_size(int vocab) { return (vocab + kChunk - 1) / kChunk; }

cudaError_t launch_ngram_topk(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                              const int32_t *hist_len, int rows, int vocab, int n, int window,
                              int k, int mask_in_place, const float *uniform, float temperature,
                              int32_t *top_idx, float *top_val, int32_t *token, int *err,
                              cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const int C = topk_cluster_size(vocab);
  void (*kernel)(TopkArgs) = k == 1 ? ngram_top1_kernel : ngram_topk_kernel;
  if (C > 8) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  TopkArgs a;
  a.logits = logits;
  a.ld = ld;
  a.history = history;
  a.hist_ld = hist_ld;
  a.hist_len = hist_len;
  a.rows = rows;
  a.vocab = vocab;
  a.n = n;
  a.window = window;
  a.k = k;
  a.mask_in_place = mask_in_place;
  a.uniform = uniform;
  a.inv_temp_log2e = 1.4426950408889634f / temperature;
  a.top_idx = top_idx;
  a.top_val = top_val;
  a.token = token;
  a.err = err;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)(rows * C));
  lc.blockDim = dim3(kThreads);
  // the history (and for k > 1 the candidate buffer in front of it)
  const size_t hist_bytes = (size_t)(window > 0 ? window : 1) * sizeof(int32_t);
  lc.dynamicSmemBytes = k == 1 ? hist_bytes : (size_t)kTopkCandidates * 8 + hist_bytes;
  if (k > 1 && lc.dynamicSmemBytes > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(ngram_topk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lc.dynamicSmemBytes);
    if (e != cudaSuccess) return e;
  }
  lc.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 2;
  return cudaLaunchKernelEx(&lc, kernel, a);
}

}  // namespace rswa
