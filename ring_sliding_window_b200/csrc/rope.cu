// Rotary position embedding (RoPE) at cache-write time.
//
// The pages ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.1) fix
// the cache -- the prompt plus a ring of the W latest generated tokens, with
// max_position_embeddings = 32768 -- but say nothing about which position a
// generated token takes once the ring has wrapped.  The library offers two
// explicit policies (rswa_rope_policy): the token's absolute position
// P_b + t, or the cache slot it is written to, P_b + (t mod W).  Keys are
// rotated once, when they enter the cache, and the cache holds rotated keys;
// queries are rotated when they are used.
//
// The rotation is the rotate-half form used by Llama-family models: for
// i < d/2 the pair (x_i, x_{i+d/2}) turns by the angle pos * theta^(-2i/d).
// Angles are formed and reduced in double precision (pos * theta^(-2i/d)
// reaches 10^6 radians, far beyond what single precision resolves) and the
// cosines and sines rounded to float; the rotation itself runs in float.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace rswa {
namespace {

__device__ __forceinline__ float2 rope_cs(int64_t pos, int i, int d, float theta) {
  const double inv_freq = pow((double)theta, -2.0 * (double)i / (double)d);
  double sn, cs;
  sincos((double)pos * inv_freq, &sn, &cs);
  return make_float2((float)cs, (float)sn);
}

// One CTA per run of kRun consecutive prompt positions of one sequence.
// Thread i < d/2 reduces the run's first angle for pair i once (double
// sincos) and walks the run with the angle-addition recurrence in double
// precision (kRun steps add a few 1e-16), leaving float (cos, sin) in shared
// memory; then all threads rotate q and k of every head of the run, each
// thread 16 bytes of both halves of a row at a time, consecutive threads on
// consecutive 16-byte pieces.
constexpr int kRun = 64;

template <typename T>
__global__ void __launch_bounds__(256)
    rope_prefill_kernel(const DeviceView v, const T *__restrict__ q, const T *__restrict__ k,
                        T *__restrict__ qr, T *__restrict__ kc) {
  __shared__ float2 cs[kRun][64];
  const int half = v.D / 2;
  const int run = blockIdx.x;
  int lo = 0, hi = v.B;  // sequence of the run: tile64_base[lo] <= run < tile64_base[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (v.tile64_base[mid] <= run) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int P = v.plen[b];
  const int p0 = (run - v.tile64_base[b]) * kRun;
  const int n = min(kRun, P - p0);
  const int i = threadIdx.x;
  if (i < half) {
    const double inv_freq = pow((double)v.rope_theta, -2.0 * (double)i / (double)v.D);
    double sn, c, sd, cd;
    sincos((double)p0 * inv_freq, &sn, &c);
    sincos(inv_freq, &sd, &cd);
    for (int j = 0; j < n; ++j) {
      cs[j][i] = make_float2((float)c, (float)sn);
      const double cn = c * cd - sn * sd;  // angle + inv_freq
      sn = sn * cd + c * sd;
      c = cn;
    }
  }
  __syncthreads();
  // one item = 16 bytes of a half row (8 bf16 or 4 fp32 pairs) of one head
  constexpr int VW = Chunk<T>::N;
  const int cph = half / VW;  // items per half row
  const int per_pos = v.H * cph;
  const int64_t tok0 = v.tok_base[b] + p0;
  const int64_t krow0 = (int64_t)v.H * v.slot_base[b] + p0;
  for (int e = threadIdx.x; e < n * per_pos; e += blockDim.x) {
    const int j = e / per_pos;
    const int rem = e - j * per_pos;
    const int h = rem / cph, ii = (rem - h * cph) * VW;
    const int64_t src = ((tok0 + j) * v.H + h) * v.D + ii;
    const int64_t dst = (krow0 + (int64_t)h * (P + v.W) + j) * v.D + ii;
    float qa[VW], qb[VW], ka[VW], kb[VW];
    Chunk<T>::widen(*reinterpret_cast<const uint4 *>(q + src), qa);
    Chunk<T>::widen(*reinterpret_cast<const uint4 *>(q + src + half), qb);
    Chunk<T>::widen(*reinterpret_cast<const uint4 *>(k + src), ka);
    Chunk<T>::widen(*reinterpret_cast<const uint4 *>(k + src + half), kb);
    float q1[VW], q2[VW], k1[VW], k2[VW];
#pragma unroll
    for (int t = 0; t < VW; ++t) {
      const float2 r = cs[j][ii + t];
      q1[t] = qa[t] * r.x - qb[t] * r.y;
      q2[t] = qb[t] * r.x + qa[t] * r.y;
      k1[t] = ka[t] * r.x - kb[t] * r.y;
      k2[t] = kb[t] * r.x + ka[t] * r.y;
    }
    *reinterpret_cast<uint4 *>(qr + src) = Chunk<T>::narrow(q1);
    *reinterpret_cast<uint4 *>(qr + src + half) = Chunk<T>::narrow(q2);
    *reinterpret_cast<uint4 *>(kc + dst) = Chunk<T>::narrow(k1);
    *reinterpret_cast<uint4 *>(kc + dst + half) = Chunk<T>::narrow(k2);
  }
}

// (cos, sin) at the position of each request's next generated token.
__global__ void rope_table_kernel(const DeviceView v) {
  const int half = v.D / 2;
  const int b = blockIdx.x;
  const int64_t t = v.t[b];
  const int64_t P = v.plen[b];
  const int64_t pos = v.rope == RSWA_ROPE_SLOT ? P + t % v.W : P + t;
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    v.rope_cs[(int64_t)b * half + i] = rope_cs(pos, i, v.D, v.rope_theta);
}

// rswa_advance with RoPE on: t_b += 1, then the table for the new position.
__global__ void advance_rope_kernel(const DeviceView v) {
  grid_dependency_wait();  // the decode kernels before it read t and the table
  allow_dependents();
  const int half = v.D / 2;
  const int b = blockIdx.x;
  const int64_t t = v.t[b] + 1;
  const int64_t P = v.plen[b];
  __syncthreads();  // every thread has read the old t
  if (threadIdx.x == 0) v.t[b] = t;
  const int64_t pos = v.rope == RSWA_ROPE_SLOT ? P + t % v.W : P + t;
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    v.rope_cs[(int64_t)b * half + i] = rope_cs(pos, i, v.D, v.rope_theta);
}

}  // namespace

cudaError_t launch_rope_prefill(const DeviceView &v, const void *q, const void *k, void *qr,
                                void *kc, cudaStream_t s) {
  if (v.total_tokens == 0) return cudaSuccess;
  static_assert(kRun == kSimtTile, "runs are counted by the 64-token tile table");
  const int grid = v.total_tiles64;
  if (v.dtype == RSWA_BF16)
    rope_prefill_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        v, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (__nv_bfloat16 *)qr,
        (__nv_bfloat16 *)kc);
  else
    rope_prefill_kernel<float><<<grid, 256, 0, s>>>(v, (const float *)q, (const float *)k,
                                                    (float *)qr, (float *)kc);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(const DeviceView &v, cudaStream_t s) {
  if (!v.rope) return cudaSuccess;
  rope_table_kernel<<<v.B, 64, 0, s>>>(v);
  return cudaGetLastError();
}

cudaError_t launch_advance_rope(const DeviceView &v, cudaStream_t s) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)v.B);
  lc.blockDim = dim3(64);
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, advance_rope_kernel, v);
}

}  // namespace rswa
