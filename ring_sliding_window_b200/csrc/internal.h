// Internal declarations shared by the librswa host layer and its kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <vector>

#include "../../include/rswa.h"

namespace rswa {

// Split-K piece of the decode attention: keys [key_begin, key_end) of one
// (b, h) ring, all processed by one CTA.  Pieces are listed in flattened
// (b, h, key) order, so the pieces of one (b, h) are contiguous.  A piece
// carries everything the kernel needs to start streaming, so one load of it
// (made before the kernel's grid-dependency wait) replaces a chain of table
// lookups.
struct __align__(16) DecodePiece {
  int64_t row0;       // cache row of slot 0 of ring (b, h), in rows of d elements
  int32_t b, h;
  int32_t key_begin, key_end;
  int32_t plen;       // P_b
  int32_t first;      // first piece of this (b, h)
  int32_t count;      // pieces of this (b, h)
  int32_t cta;
};

// Byte offsets of the workspace sections (each 256-byte aligned).
struct WsLayout {
  size_t err;        // int32 device error word (+ int32 debug flags)
  size_t t;          // int64 [B]   tokens generated so far
  size_t plen;       // int32 [B]   P_b
  size_t slot_base;  // int64 [B+1] first cache slot of each request
  size_t tok_base;   // int64 [B+1] sum_{b'<b} P_b'
  size_t tile_base;  // int32 [B+1] sum_{b'<b} ceil(P_b' / kPrefillTile)
  size_t tile64_base;  // int32 [B+1] sum_{b'<b} ceil(P_b' / kSimtTile)
  size_t pf_blocks;  // int4 [n_pf_blocks] (b, h, first query tile, tiles 1|2)
  size_t pieces;     // DecodePiece [n_pieces]
  size_t cta_piece;  // int32 [G+1] first piece of each decode CTA
  size_t bh_piece;   // int32 [B*H+1] first piece of each (b, h)
  size_t bh_count;   // int32 [B*H]   pieces of (b, h) finished in this launch
  size_t part_ml;    // float2 [n_pieces] (running max in log2 units, sum)
  size_t part_o;     // float [n_pieces][d] unnormalised outputs
  size_t rope_cs;    // float2 [B][d/2] (cos, sin) at each request's current position
  size_t total;
};

// Host-side plan of the decode decomposition (depends on the SM count).
struct DecodePlan {
  int grid;      // decode CTAs
  int n_pieces;  // total pieces
  std::vector<DecodePiece> pieces;
  std::vector<int32_t> cta_piece;  // [grid + 1]
  std::vector<int32_t> bh_piece;   // [B*H + 1]
};

constexpr int kTopkMax = 64;                 // largest k of rswa_ngram_topk
constexpr int kTopkMaxVocab = 16 * 16384;    // 16 CTAs of 16,384 columns per row
constexpr int kTopkMaxWindow = 8192;         // history staged in shared memory
constexpr int kPrefillTile = 128;  // query rows per prefill tile (tensor-core kernel)
constexpr int kSimtTile = 64;      // query rows per prefill tile (FP32 SIMT kernel)

// Everything the kernels need, as plain device pointers.
struct DeviceView {
  int B, H, D, W, L;
  int dtype;
  float scale;
  int *err;
  const int *fault;  // fault-injection flags (tests only; 0 in normal use)
  int64_t *t;
  const int32_t *plen;
  const int64_t *slot_base;
  const int64_t *tok_base;
  const int32_t *tile_base;
  const int32_t *tile64_base;
  const int4 *pf_blocks;
  int n_pf_blocks;
  const DecodePiece *pieces;
  const int32_t *cta_piece;
  const int32_t *bh_piece;
  int *bh_count;
  float2 *part_ml;
  float *part_o;
  int decode_grid;
  int n_pieces;
  int cluster_size;  // > 0: decode runs one ring per cluster of this many CTAs
  int swa;           // 1: standard sliding window (the window also cuts the prompt)
  int key_lo, key_hi;  // slot range a decode step attends to (a share of a split cache)
  float2 *out_ml;      // non-null: write (m, l) [B*H] and o [B*H][D] instead of out
  float *out_o;
  int rope;          // rswa_rope_policy (0: keys and queries used as given)
  float rope_theta;
  float2 *rope_cs;   // [B][D/2] (cos, sin) of the position of each request's next token
  int64_t total_tokens;  // sum P_b
  int total_tiles;       // sum ceil(P_b / kPrefillTile)
  int total_tiles64;     // sum ceil(P_b / kSimtTile)
  int max_plen;
};

}  // namespace rswa

struct rswa_state {
  rswa_config cfg;
  std::vector<int64_t> plen;
  std::vector<int64_t> slot_base;  // first cache slot of each request
  int64_t pool_slots;              // slots the caches hold (per layer, K or V)
  std::vector<void *> k_cache, v_cache;
  std::vector<uint8_t> layer_ready;  // prefilled or resumed
  void *workspace;
  size_t workspace_size;
  int device;
  int num_sms;
  rswa::WsLayout ws;
  rswa::DecodePlan plan;
  rswa::DeviceView dv;
};

namespace rswa {

// Launchers (return cudaGetLastError() of their launch).
// pdl: launch with programmatic stream serialization (the kernel waits for
// the previous kernel's completion before touching any produced data).
cudaError_t launch_decode(const DeviceView &v, const void *q, const void *k_new,
                          const void *v_new, void *kc, void *vc, void *out, cudaStream_t s,
                          bool pdl);
cudaError_t launch_advance(const DeviceView &v, cudaStream_t s);
cudaError_t launch_combine(const float2 *ml, const float *o, int shares, int64_t rings, int D,
                           int dtype, void *out, cudaStream_t s);
cudaError_t launch_ngram_topk(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                              const int32_t *hist_len, int rows, int vocab, int n, int window,
                              int k, int mask_in_place, const float *uniform, float temperature,
                              int32_t *top_idx, float *top_val, int32_t *token, int *err,
                              cudaStream_t s);
cudaError_t launch_cache_fill(const DeviceView &v, const void *k, const void *vv, void *kc,
                              void *vc, cudaStream_t s);
// RoPE of the prompt: rotated k into cache slots [0, P_b), rotated q into `qr`.
cudaError_t launch_rope_prefill(const DeviceView &v, const void *q, const void *k, void *qr,
                                void *kc, cudaStream_t s);
// (cos, sin) table of every request's next-token position (v.rope_cs).
cudaError_t launch_rope_table(const DeviceView &v, cudaStream_t s);
cudaError_t launch_advance_rope(const DeviceView &v, cudaStream_t s);
// kc: NULL to read K from `k`; else K is read from this layer's cache
// (rotated keys, RoPE), which holds kc_rows rows of d elements.
cudaError_t launch_prefill_simt(const DeviceView &v, const void *q, const void *k,
                                const void *vv, void *out, const void *kc, cudaStream_t s);
// The bf16 d = 128 prefill on the tensor cores.  It also fills cache slots
// [0, P_b) of kc / vc (which hold kc_rows rows of d elements) with the
// prompt's K / V; k_from_cache: K is read from kc (rotated keys, RoPE) and
// only V is stored.
cudaError_t launch_prefill_tc(const DeviceView &v, const void *q, const void *k, const void *vv,
                              void *out, const int4 *blocks, int n_blocks, void *kc, void *vc,
                              int k_from_cache, int64_t kc_rows, cudaStream_t s);

// Prefill work list of the tensor-core kernel: blocks of two consecutive
// 128-row query tiles of one (b, h), in launch order.
// one_tile: one query tile per block (the standard sliding window's blocks
// have different key ranges per tile).
std::vector<int4> plan_prefill_blocks(const rswa_config *c, const int64_t *plen, int num_sms,
                                      bool one_tile = false);
cudaError_t launch_ngram(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                         const int32_t *hist_len, int rows, int vocab, int n, int window,
                         int *err, cudaStream_t s);

// Resident decode CTAs per SM for (dtype, head_dim); used by the planner.
int decode_ctas_per_sm(int dtype, int head_dim);
// Clusters of `cluster` decode CTAs that can be resident at once (0: none).
int decode_max_clusters(int dtype, int head_dim, int cluster);

// Host-side helpers of the planner (rswa_api.cu).
bool config_ok(const rswa_config *c, const int64_t *plen);
int current_device();
int sm_count(int dev);
// slot_base: host [B] first cache slot of each request, or NULL for requests
// packed back to back in batch order.
DecodePlan plan_decode(const rswa_config *c, const int64_t *plen, const int64_t *slot_base,
                       int num_sms, int ctas_per_sm);
WsLayout layout_ws(const rswa_config *c, const int64_t *plen, const DecodePlan &p);

}  // namespace rswa
