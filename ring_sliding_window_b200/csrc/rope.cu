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

// One thread per (prompt token, pair i): the angle is computed once and
// applied to q and k of every head.
template <typename T>
__global__ void rope_prefill_kernel(const DeviceView v, const T *__restrict__ q,
                                    const T *__restrict__ k, T *__restrict__ qr,
                                    T *__restrict__ kc) {
  const int half = v.D / 2;
  const int64_t total = v.total_tokens * half;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tk = w / half;
    const int i = (int)(w % half);
    int lo = 0, hi = v.B;  // sequence of token tk: tok_base[lo] <= tk < tok_base[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (v.tok_base[mid] <= tk) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int64_t slot = tk - v.tok_base[b];  // = the prompt position
    const int P = v.plen[b];
    const float2 cs = rope_cs(slot, i, v.D, v.rope_theta);
    for (int h = 0; h < v.H; ++h) {
      const int64_t src = (tk * v.H + h) * v.D;
      const int64_t drow = ((int64_t)v.H * v.slot_base[b] + (int64_t)h * (P + v.W) + slot) * v.D;
      const float qa = to_float(q[src + i]), qb = to_float(q[src + i + half]);
      const float ka = to_float(k[src + i]), kb = to_float(k[src + i + half]);
      qr[src + i] = from_float<T>(qa * cs.x - qb * cs.y);
      qr[src + i + half] = from_float<T>(qb * cs.x + qa * cs.y);
      kc[drow + i] = from_float<T>(ka * cs.x - kb * cs.y);
      kc[drow + i + half] = from_float<T>(kb * cs.x + ka * cs.y);
    }
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

int grid_for(int64_t work, int threads) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (work + threads - 1) / threads;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_rope_prefill(const DeviceView &v, const void *q, const void *k, void *qr,
                                void *kc, cudaStream_t s) {
  if (v.total_tokens == 0) return cudaSuccess;
  const int threads = 256;
  const int grid = grid_for(v.total_tokens * (v.D / 2), threads);
  if (v.dtype == RSWA_BF16)
    rope_prefill_kernel<__nv_bfloat16><<<grid, threads, 0, s>>>(
        v, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (__nv_bfloat16 *)qr,
        (__nv_bfloat16 *)kc);
  else
    rope_prefill_kernel<float><<<grid, threads, 0, s>>>(v, (const float *)q, (const float *)k,
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
