// Allocation-free variant of the decode step.
//
// rswa_decode_step needs a caller-allocated workspace (work tables, ring
// counters and the split-K partials).  Some callers cannot provide one at the
// point where they decode: a plugin hosted by another runtime or inference
// server receives its input and output tensors but must not allocate device
// memory itself (the host application's allocator already owns the pool, so a
// private cudaMalloc can fail or fragment it), and a latency-bound serving
// loop must keep cudaMalloc/cudaFree off its hot path because both can
// synchronise the device and stall every other stream.
//
// rswa_decode_step_noalloc serves them: it runs the same split-K kernels as
// rswa_decode_step, with the scratch taken from a file-scope __device__ array
// of a fixed size (kNoAllocScratchBytes per device, held until the process
// exits).  The caller still passes the cache, inputs and outputs.
#include <climits>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "internal.h"

namespace rswa {
namespace {

constexpr size_t kNoAllocScratchBytes = RSWA_NOALLOC_SCRATCH_BYTES;

// Shared by every call on a device.  Host code must not use this name as an
// address: the device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for `dev` (the current device), looked
// up once per device.
rswa_status scratch_for_device(int dev, uint8_t **out) {
  if (dev < 0 || dev >= kMaxDevices) return RSWA_EINVAL;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RSWA_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = (uint8_t *)g_scratch_ptr[dev];
  return RSWA_OK;
}

// Resident decode CTAs per SM for (device, dtype, head_dim), worked out once:
// the query sets a function attribute and runs an occupancy calculation,
// which a latency-bound serving loop should not repeat at every step.
int g_ctas_per_sm[kMaxDevices][4] = {};

int ctas_per_sm_cached(int dev, int dtype, int head_dim) {
  const int key = (dtype == RSWA_BF16 ? 0 : 2) + (head_dim == 128 ? 0 : 1);
  std::lock_guard<std::mutex> lock(g_setup_mu);
  int &n = g_ctas_per_sm[dev][key];
  if (n == 0) n = decode_ctas_per_sm(dtype, head_dim);
  return n;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Sections of the array that the decode kernel reads or writes, in the
// workspace's order.  Only these count against the limit: the prefill and
// RoPE tables of a full workspace are never touched by a decode step.
struct NoAllocLayout {
  size_t err, t, plen, slot_base, pieces, cta_piece, bh_piece, bh_count, part_ml, part_o, total;
};

NoAllocLayout noalloc_layout(const rswa_config *c, const DecodePlan &p) {
  const size_t B = (size_t)c->batch, BH = B * (size_t)c->num_heads;
  NoAllocLayout w;
  size_t off = 0;
  w.err = off;       off = align256(off + 2 * sizeof(int32_t));  // error word, fault flags
  w.t = off;         off = align256(off + 2 * B * sizeof(int64_t));
  w.plen = off;      off = align256(off + B * sizeof(int32_t));
  w.slot_base = off; off = align256(off + (B + 1) * sizeof(int64_t));
  w.pieces = off;    off = align256(off + (size_t)p.n_pieces * sizeof(DecodePiece));
  w.cta_piece = off; off = align256(off + ((size_t)p.grid + 1) * sizeof(int32_t));
  w.bh_piece = off;  off = align256(off + (BH + 1) * sizeof(int32_t));
  w.bh_count = off;  off = align256(off + BH * sizeof(int32_t));
  w.part_ml = off;   off = align256(off + (size_t)p.n_pieces * sizeof(float2));
  w.part_o = off;    off = align256(off + (size_t)p.n_pieces * c->head_dim * sizeof(float));
  w.total = off;
  return w;
}

// The work tables travel to the array inside kernel parameters: the launch
// copies its parameters when it is enqueued, so nothing refers to the
// caller's (or this call's) host memory once the call has returned.
constexpr int kUploadChunk = 16384;
struct __align__(16) UploadChunk {
  uint8_t bytes[kUploadChunk];
};

__global__ void __launch_bounds__(256) noalloc_upload_kernel(uint8_t *dst,
                                                             const __grid_constant__ UploadChunk c,
                                                             int n16) {
  const uint4 *src = reinterpret_cast<const uint4 *>(c.bytes);
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  for (int i = threadIdx.x; i < n16; i += blockDim.x) d[i] = src[i];
}

}  // namespace
}  // namespace rswa

using namespace rswa;

extern "C" rswa_status rswa_decode_step_noalloc(const rswa_config *cfg,
                                                const int64_t *prefill_len,
                                                const int64_t *n_generated, void *k_cache,
                                                void *v_cache, const void *q, const void *k_new,
                                                const void *v_new, void *out,
                                                int32_t *device_error, void *stream) {
  if (!config_ok(cfg, prefill_len) || !n_generated) return RSWA_EINVAL;
  if (!k_cache || !v_cache || !q || !k_new || !v_new || !out) return RSWA_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(k_new) ||
      !aligned16(v_new) || !aligned16(out))
    return RSWA_EINVAL;
  const int B = cfg->batch;
  for (int b = 0; b < B; ++b)
    if (n_generated[b] < 0) return RSWA_EINVAL;
  const int dev = current_device();
  if (dev < 0) return RSWA_ECUDA;
  if (dev >= kMaxDevices) return RSWA_EINVAL;

  const DecodePlan plan = plan_decode(cfg, prefill_len, nullptr, sm_count(dev),
                                      ctas_per_sm_cached(dev, cfg->dtype, cfg->head_dim));
  const NoAllocLayout ws = noalloc_layout(cfg, plan);
  if (ws.total > kNoAllocScratchBytes) return RSWA_ENOMEM;  // batch too large for the array

  uint8_t *scratch = nullptr;
  const rswa_status st = scratch_for_device(dev, &scratch);
  if (st != RSWA_OK) return st;

  // Host image of the tables.  The error word and the per-(b, h) completion
  // counters in it are zero, so every call starts from cleared values; the
  // partials are fully overwritten by the split kernel and need no clearing.
  // part_ml is 256-byte aligned, so the image is a whole number of 16-byte
  // words.
  std::vector<uint8_t> img(ws.part_ml, 0);
  int64_t *t = (int64_t *)(img.data() + ws.t);
  int32_t *pl = (int32_t *)(img.data() + ws.plen);
  int64_t *sb = (int64_t *)(img.data() + ws.slot_base);
  for (int b = 0; b < B; ++b) {
    t[b] = n_generated[b];
    t[B + b] = n_generated[b];
    pl[b] = (int32_t)prefill_len[b];
    sb[b + 1] = sb[b] + prefill_len[b] + cfg->window;
  }
  memcpy(img.data() + ws.pieces, plan.pieces.data(), plan.pieces.size() * sizeof(DecodePiece));
  memcpy(img.data() + ws.cta_piece, plan.cta_piece.data(), plan.cta_piece.size() * sizeof(int32_t));
  memcpy(img.data() + ws.bh_piece, plan.bh_piece.data(), plan.bh_piece.size() * sizeof(int32_t));
  cudaStream_t s = (cudaStream_t)stream;
  UploadChunk chunk;
  for (size_t off = 0; off < img.size(); off += kUploadChunk) {
    const size_t n = std::min(img.size() - off, (size_t)kUploadChunk);
    memcpy(chunk.bytes, img.data() + off, n);
    noalloc_upload_kernel<<<1, 256, 0, s>>>(scratch + off, chunk, (int)(n / 16));
    if (cudaGetLastError() != cudaSuccess) return RSWA_ECUDA;
  }

  DeviceView v;
  memset(&v, 0, sizeof(v));
  v.key_hi = INT_MAX;  // the whole cache
  v.B = B;
  v.H = cfg->num_heads;
  v.D = cfg->head_dim;
  v.W = cfg->window;
  v.L = 1;
  v.dtype = cfg->dtype;
  v.scale = cfg->scale == 0.f ? 1.0f / sqrtf((float)cfg->head_dim) : cfg->scale;
  v.err = device_error ? (int *)device_error : (int *)(scratch + ws.err);
  v.fault = (const int *)(scratch + ws.err) + 1;  // zero: the table image clears it
  v.t = (int64_t *)(scratch + ws.t);
  v.plen = (const int32_t *)(scratch + ws.plen);
  v.slot_base = (const int64_t *)(scratch + ws.slot_base);
  v.pieces = (const DecodePiece *)(scratch + ws.pieces);
  v.cta_piece = (const int32_t *)(scratch + ws.cta_piece);
  v.bh_piece = (const int32_t *)(scratch + ws.bh_piece);
  v.bh_count = (int *)(scratch + ws.bh_count);
  v.part_ml = (float2 *)(scratch + ws.part_ml);
  v.part_o = (float *)(scratch + ws.part_o);
  v.decode_grid = plan.grid;
  v.n_pieces = plan.n_pieces;
  // Plain launch (no programmatic dependent launch): the table upload
  // kernels just before it must be complete when it starts.
  return launch_decode(v, q, k_new, v_new, k_cache, v_cache, out, s, false) == cudaSuccess
             ? RSWA_OK
             : RSWA_ECUDA;
}
