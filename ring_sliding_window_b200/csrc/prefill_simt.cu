// Prefill on CUDA cores (FP32 FMA), and the prefill cache fill.
//
// Method ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.1): the
// prefill segment keeps full attention -- every prompt token attends causally
// to all earlier prompt tokens and every prompt K/V stays in the cache.
//
// prefill_simt_kernel is the fp32 path (fp32 inputs must meet a 1e-5 bound,
// which TF32 tensor cores cannot): a flash-style loop over 64-key tiles staged
// in shared memory as fp32, online softmax in the log2 domain, one query row
// per D/32 threads (each thread owns 32 interleaved elements of q and of the
// output accumulator).  It also accepts bf16 inputs.
//
// cache_fill_kernel copies the packed prompt K/V [sum P][H][d] into cache
// slots [0, P_b) of the head-major cache, 16 bytes per thread.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace rswa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// index b with base[b] <= x < base[b+1]; base has B+1 entries, base[0] == 0
template <typename I>
__device__ __forceinline__ int find_seq(const I *base, int B, int64_t x) {
  int lo = 0, hi = B;  // invariant: base[lo] <= x < base[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)base[mid] <= x)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

template <typename T, int D>
struct SimtShape {
  static constexpr int kTPR = D / 32;               // threads per query row
  static constexpr int kRows = kSimtTile;           // query rows per CTA
  static constexpr int kKeys = 64;                  // keys per staged tile
  static constexpr int kThreads = kRows * kTPR;
  static constexpr int kChunks = D / 4;             // float4 chunks per fp32 row
  static constexpr int kChunksPerThread = kChunks / kTPR;  // 8
  static constexpr int kSub = 8;                    // keys per online-softmax chunk
};

template <typename T, int D>
__global__ void __launch_bounds__(SimtShape<T, D>::kThreads)
    prefill_simt_kernel(const DeviceView v, const T *q, const T *__restrict__ k,
                        const T *__restrict__ vv, T *out, const T *__restrict__ kc) {
  using S = SimtShape<T, D>;
  extern __shared__ __align__(16) float smem_f[];
  float *Ks = smem_f;                 // [kKeys][D]
  float *Vs = smem_f + S::kKeys * D;  // [kKeys][D]

  const int h = blockIdx.y;
  const int tile = blockIdx.x;
  const int b = find_seq(v.tile64_base, v.B, tile);
  const int qt = tile - v.tile64_base[b];  // tile index inside the sequence
  const int P = v.plen[b];
  const int64_t tok0 = v.tok_base[b];
  const int HD = v.H * D;
  // K rows from the cache (rotated keys) when kc is given
  const int64_t krow0 = (int64_t)v.H * v.slot_base[b] + (int64_t)h * (P + v.W);

  const int row = threadIdx.x / S::kTPR;
  const int sub = threadIdx.x % S::kTPR;
  const int qi = qt * S::kRows + row;  // query position inside the sequence
  const bool row_ok = qi < P;

  float qf[S::kChunksPerThread * 4];
  float o[S::kChunksPerThread * 4];
  const float qs = v.scale * kLog2e;
#pragma unroll
  for (int j = 0; j < S::kChunksPerThread; ++j) {
    const int c = sub + S::kTPR * j;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      qf[4 * j + e] = row_ok ? to_float(q[(tok0 + qi) * HD + h * D + 4 * c + e]) * qs : 0.f;
      o[4 * j + e] = 0.f;
    }
  }
  float m = -INFINITY, l = 0.f;

  const int last_key = min(qt * S::kRows + S::kRows, P);  // keys [0, last_key) may be needed
  // standard sliding window: query qi sees keys (qi - W, qi] only
  const int first_key = v.swa ? max(0, qt * S::kRows - v.W + 1) / S::kKeys * S::kKeys : 0;
  for (int k0 = first_key; k0 < last_key; k0 += S::kKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < S::kKeys * D; idx += S::kThreads) {
      const int r = idx / D, e = idx % D;
      const int kj = k0 + r;
      float kx = 0.f, vx = 0.f;
      if (kj < P) {
        const int64_t off = (tok0 + kj) * HD + h * D + e;
        kx = to_float(kc ? kc[(krow0 + kj) * D + e] : k[off]);
        vx = to_float(vv[off]);
      }
      Ks[idx] = kx;
      Vs[idx] = vx;
    }
    __syncthreads();
    const int kend = min(S::kKeys, P - k0);
    for (int j0 = 0; j0 < kend; j0 += S::kSub) {
      float sc[S::kSub];
#pragma unroll
      for (int jj = 0; jj < S::kSub; ++jj) {
        const int kr = j0 + jj;
        const float4 *krow = reinterpret_cast<const float4 *>(Ks + kr * D);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < S::kChunksPerThread; ++j) {
          const float4 kk = krow[sub + S::kTPR * j];
          acc = fmaf(qf[4 * j], kk.x, acc);
          acc = fmaf(qf[4 * j + 1], kk.y, acc);
          acc = fmaf(qf[4 * j + 2], kk.z, acc);
          acc = fmaf(qf[4 * j + 3], kk.w, acc);
        }
#pragma unroll
        for (int x = 1; x < S::kTPR; x <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, x);
        const int kpos = k0 + kr;
        sc[jj] = (row_ok && kr < kend && kpos <= qi && (!v.swa || kpos > qi - v.W)) ? acc
                                                                                    : -INFINITY;
      }
      float m_new = m;
#pragma unroll
      for (int jj = 0; jj < S::kSub; ++jj) m_new = fmaxf(m_new, sc[jj]);
      if (m_new == -INFINITY) continue;
      const float corr = exp2f(m - m_new);
      l *= corr;
#pragma unroll
      for (int e = 0; e < S::kChunksPerThread * 4; ++e) o[e] *= corr;
#pragma unroll
      for (int jj = 0; jj < S::kSub; ++jj) {
        const float p = exp2f(sc[jj] - m_new);
        l += p;
        const float4 *vrow = reinterpret_cast<const float4 *>(Vs + (j0 + jj) * D);
#pragma unroll
        for (int j = 0; j < S::kChunksPerThread; ++j) {
          const float4 x = vrow[sub + S::kTPR * j];
          o[4 * j] = fmaf(p, x.x, o[4 * j]);
          o[4 * j + 1] = fmaf(p, x.y, o[4 * j + 1]);
          o[4 * j + 2] = fmaf(p, x.z, o[4 * j + 2]);
          o[4 * j + 3] = fmaf(p, x.w, o[4 * j + 3]);
        }
      }
      m = m_new;
    }
  }
  if (row_ok) {
    const float inv = 1.f / l;
#pragma unroll
    for (int j = 0; j < S::kChunksPerThread; ++j) {
      const int c = sub + S::kTPR * j;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        out[(tok0 + qi) * HD + h * D + 4 * c + e] = from_float<T>(o[4 * j + e] * inv);
    }
  }
}

// Copy prompt K/V into cache slots [0, P_b).  One 16-byte chunk per thread
// iteration; chunks of a token row are contiguous on both sides per head.
template <int ROW_BYTES>
__global__ void cache_fill_kernel(const DeviceView v, const uint8_t *__restrict__ k,
                                  const uint8_t *__restrict__ vv, uint8_t *kc, uint8_t *vc) {
  constexpr int kChunks = ROW_BYTES / 16;
  const int64_t total = v.total_tokens * v.H * kChunks;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < total;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tk = c / (v.H * kChunks);
    const int rem = (int)(c % (v.H * kChunks));
    const int h = rem / kChunks, ch = rem % kChunks;
    const int b = find_seq(v.tok_base, v.B, tk);
    const int64_t slot = tk - v.tok_base[b];
    const int P = v.plen[b];
    const int64_t drow = (int64_t)v.H * v.slot_base[b] + (int64_t)h * (P + v.W) + slot;
    const int64_t src = c * 16;
    const int64_t dst = drow * ROW_BYTES + ch * 16;
    *reinterpret_cast<uint4 *>(kc + dst) = *reinterpret_cast<const uint4 *>(k + src);
    *reinterpret_cast<uint4 *>(vc + dst) = *reinterpret_cast<const uint4 *>(vv + src);
  }
}

template <typename T, int D>
cudaError_t launch_simt_t(const DeviceView &v, const void *q, const void *k, const void *vv,
                          void *out, const void *kc, cudaStream_t s) {
  using S = SimtShape<T, D>;
  const int smem = 2 * S::kKeys * D * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(v.total_tiles64, v.H);
  prefill_simt_kernel<T, D><<<grid, S::kThreads, smem, s>>>(v, (const T *)q, (const T *)k,
                                                            (const T *)vv, (T *)out,
                                                            (const T *)kc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const DeviceView &v, const void *q, const void *k,
                                const void *vv, void *out, const void *kc, cudaStream_t s) {
  if (v.total_tiles64 == 0) return cudaSuccess;
  if (v.dtype == RSWA_BF16)
    return v.D == 128 ? launch_simt_t<__nv_bfloat16, 128>(v, q, k, vv, out, kc, s)
                      : launch_simt_t<__nv_bfloat16, 64>(v, q, k, vv, out, kc, s);
  return v.D == 128 ? launch_simt_t<float, 128>(v, q, k, vv, out, kc, s)
                    : launch_simt_t<float, 64>(v, q, k, vv, out, kc, s);
}

cudaError_t launch_cache_fill(const DeviceView &v, const void *k, const void *vv, void *kc,
                              void *vc, cudaStream_t s) {
  if (v.total_tokens == 0) return cudaSuccess;
  const int row_bytes = v.D * (v.dtype == RSWA_BF16 ? 2 : 4);
  const int64_t chunks = v.total_tokens * v.H * (row_bytes / 16);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (chunks + 255) / 256;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  const uint8_t *kb = (const uint8_t *)k, *vb = (const uint8_t *)vv;
  uint8_t *kcb = (uint8_t *)kc, *vcb = (uint8_t *)vc;
  switch (row_bytes) {
    case 128: cache_fill_kernel<128><<<(int)blocks, 256, 0, s>>>(v, kb, vb, kcb, vcb); break;
    case 256: cache_fill_kernel<256><<<(int)blocks, 256, 0, s>>>(v, kb, vb, kcb, vcb); break;
    case 512: cache_fill_kernel<512><<<(int)blocks, 256, 0, s>>>(v, kb, vb, kcb, vcb); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rswa
