// librswa host layer: argument checks, the split-K work plan, the workspace
// layout, and the exported C entry points declared in include/rswa.h.
#include <climits>
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "internal.h"

using namespace rswa;

namespace {
constexpr int64_t kMinRowsPerCta = 64;  // below this a decode CTA is mostly latency
}  // namespace

namespace rswa {

bool config_ok(const rswa_config *c, const int64_t *plen) {
  if (!c || !plen) return false;
  if (c->batch < 1 || c->num_layers < 1 || c->num_heads < 1 || c->window < 1) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->dtype != RSWA_F32 && c->dtype != RSWA_BF16) return false;
  if (!(c->scale >= 0.f) || !isfinite(c->scale)) return false;
  int64_t rows = 0;
  for (int b = 0; b < c->batch; ++b) {
    if (plen[b] < 0 || plen[b] + c->window >= (int64_t(1) << 31)) return false;
    rows += (plen[b] + c->window) * c->num_heads;
    if (rows >= (int64_t(1) << 40)) return false;
  }
  return true;
}

}  // namespace rswa

namespace {

size_t elem_size(const rswa_config *c) { return c->dtype == RSWA_BF16 ? 2 : 4; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

namespace rswa {

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

int sm_count(int dev) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 148;
  return n;
}

// Equal contiguous ranges of the flattened (b, h, key) rows, one per CTA.
DecodePlan plan_decode(const rswa_config *c, const int64_t *plen, const int64_t *slot_base,
                       int num_sms, int ctas_per_sm) {
  const int B = c->batch, H = c->num_heads, W = c->window;
  std::vector<int64_t> base((size_t)B, 0);
  for (int b = 0; b < B; ++b)
    base[(size_t)b] = slot_base ? slot_base[b] : (b ? base[(size_t)b - 1] + plen[b - 1] + W : 0);
  std::vector<int64_t> seg_start((size_t)B * H + 1, 0);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      seg_start[(size_t)b * H + h + 1] = seg_start[(size_t)b * H + h] + plen[b] + W;
  const int64_t R = seg_start.back();
  int64_t G = std::min<int64_t>((int64_t)num_sms * ctas_per_sm, (R + kMinRowsPerCta - 1) / kMinRowsPerCta);
  if (G < 1) G = 1;
  const int64_t rpc = (R + G - 1) / G;
  G = (R + rpc - 1) / rpc;

  DecodePlan p;
  p.grid = (int)G;
  p.cta_piece.assign((size_t)G + 1, 0);
  p.bh_piece.assign((size_t)B * H + 1, 0);
  size_t seg = 0;
  for (int64_t cta = 0; cta < G; ++cta) {
    p.cta_piece[(size_t)cta] = (int32_t)p.pieces.size();
    int64_t r0 = cta * rpc;
    const int64_t r1 = std::min(R, r0 + rpc);
    while (r0 < r1) {
      while (seg_start[seg + 1] <= r0) ++seg;
      const int64_t e = std::min(r1, seg_start[seg + 1]);
      DecodePiece pc;
      pc.b = (int32_t)(seg / (size_t)H);
      pc.h = (int32_t)(seg % (size_t)H);
      pc.row0 = (int64_t)H * base[(size_t)pc.b] + (int64_t)pc.h * (plen[pc.b] + W);
      pc.key_begin = (int32_t)(r0 - seg_start[seg]);
      pc.key_end = (int32_t)(e - seg_start[seg]);
      pc.plen = (int32_t)plen[pc.b];
      pc.first = 0;
      pc.count = 0;
      pc.cta = (int32_t)cta;
      p.pieces.push_back(pc);
      r0 = e;
    }
  }
  p.cta_piece[(size_t)G] = (int32_t)p.pieces.size();
  p.n_pieces = (int)p.pieces.size();
  // first piece of each (b, h): pieces are in flattened order
  size_t i = 0;
  for (size_t bh = 0; bh <= (size_t)B * H; ++bh) {
    while (i < p.pieces.size() && (size_t)p.pieces[i].b * H + p.pieces[i].h < bh) ++i;
    p.bh_piece[bh] = (int32_t)i;
  }
  for (DecodePiece &pc : p.pieces) {
    const size_t bh = (size_t)pc.b * H + pc.h;
    pc.first = p.bh_piece[bh];
    pc.count = p.bh_piece[bh + 1] - p.bh_piece[bh];
  }
  return p;
}

// Blocks of two consecutive query tiles of one (b, h).  A block's causal work
// grows with its tile index.  (b, h) rings are taken in super-groups of about
// one wave of blocks; inside a super-group blocks run longest first.  The
// CTAs running together then share a few rings' K/V through L2, and the
// last wave is not left with one long block.
std::vector<int4> plan_prefill_blocks(const rswa_config *c, const int64_t *plen, int num_sms,
                                      bool one_tile) {
  const int B = c->batch, H = c->num_heads;
  // Pairs of tiles halve the K/V traffic per query row, but a batch too
  // small to give every SM a pair runs faster with one tile per CTA.
  int64_t pairs = 0;
  for (int b = 0; b < B; ++b) pairs += (int64_t)H * ((plen[b] + 2 * kPrefillTile - 1) / (2 * kPrefillTile));
  const int per_block = pairs >= num_sms && !one_tile ? 2 : 1;
  std::vector<int4> out;
  std::vector<int4> group, tail;
  int64_t group_blocks = 0;
  // A batch of several waves ends with the blocks of short query tiles (the
  // first eighth of every prompt's tiles), longest first: the last wave then
  // holds no long block that the other SMs would wait for.  Those blocks read
  // few K/V tiles, so losing their L2 sharing costs little.
  const bool defer = per_block == 2 && pairs >= 4 * (int64_t)num_sms;
  auto flush = [&]() {
    std::stable_sort(group.begin(), group.end(),
                     [](const int4 &x, const int4 &y) { return x.z > y.z; });
    out.insert(out.end(), group.begin(), group.end());
    group.clear();
    group_blocks = 0;
  };
  for (int b = 0; b < B; ++b) {
    const int tiles = (int)((plen[b] + kPrefillTile - 1) / kPrefillTile);
    for (int h = 0; h < H; ++h) {
      // With an odd tile count one tile has no partner, and a lone tile runs
      // at about half the rate of a pair (its softmax has no other tile's
      // MMAs to overlap).  Make that tile the first, whose single key tile
      // costs little, so the last, longest tiles are paired.
      int t0 = 0;
      if (per_block == 2 && (tiles & 1)) {
        group.push_back(make_int4(b, h, 0, 1));
        t0 = 1;
      }
      for (; t0 < tiles; t0 += per_block) {
        const int4 blk = make_int4(b, h, t0, tiles - t0 >= per_block ? per_block : 1);
        if (defer && t0 < tiles / 8)
          tail.push_back(blk);
        else
          group.push_back(blk);
      }
      group_blocks += (tiles + per_block - 1) / per_block;
      if (group_blocks >= num_sms) flush();
    }
  }
  flush();
  std::stable_sort(tail.begin(), tail.end(),
                   [](const int4 &x, const int4 &y) { return x.z > y.z; });
  out.insert(out.end(), tail.begin(), tail.end());
  return out;
}

WsLayout layout_ws(const rswa_config *c, const int64_t *plen, const DecodePlan &p) {
  const size_t B = (size_t)c->batch;
  WsLayout w;
  size_t off = 0;
  w.err = off;         off = align256(off + 2 * sizeof(int32_t));
  w.t = off;           off = align256(off + 2 * B * sizeof(int64_t));  // t and its reset copy
  w.plen = off;        off = align256(off + B * sizeof(int32_t));
  w.slot_base = off;   off = align256(off + (B + 1) * sizeof(int64_t));
  w.tok_base = off;    off = align256(off + (B + 1) * sizeof(int64_t));
  w.tile_base = off;   off = align256(off + (B + 1) * sizeof(int32_t));
  w.tile64_base = off; off = align256(off + (B + 1) * sizeof(int32_t));
  size_t blocks = 0;  // upper bound: one tile per block
  for (int b = 0; b < c->batch; ++b)
    blocks += (size_t)c->num_heads * (size_t)((plen[b] + kPrefillTile - 1) / kPrefillTile);
  w.pf_blocks = off;   off = align256(off + blocks * sizeof(int4));
  w.pieces = off;      off = align256(off + (size_t)p.n_pieces * sizeof(DecodePiece));
  w.cta_piece = off;   off = align256(off + ((size_t)p.grid + 1) * sizeof(int32_t));
  w.bh_piece = off;    off = align256(off + (B * c->num_heads + 1) * sizeof(int32_t));
  w.bh_count = off;    off = align256(off + (B * c->num_heads) * sizeof(int32_t));
  w.part_ml = off;     off = align256(off + (size_t)p.n_pieces * sizeof(float2));
  w.part_o = off;      off = align256(off + (size_t)p.n_pieces * c->head_dim * sizeof(float));
  w.rope_cs = off;     off = align256(off + B * (size_t)(c->head_dim / 2) * sizeof(float2));
  w.total = off;
  return w;
}

}  // namespace rswa

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Decode split for this batch: 0 = stream-K pieces merged through global
// memory; C > 0 = one ring per cluster of C CTAs merged through distributed
// shared memory.  The cluster form is used when every ring's cluster can be
// resident at once and gives at least half the CTAs stream-K would (small
// batches of short rings, where the global hand-off dominates).
// RSWA_DECODE_SPLIT=streamk|cluster overrides the choice (the cluster form
// still needs the clusters to fit).
int choose_cluster_size(const rswa_config *c, const int64_t *plen, int num_sms) {
  const char *env = getenv("RSWA_DECODE_SPLIT");
  const bool force_streamk = env && strcmp(env, "streamk") == 0;
  const bool force_cluster = env && strcmp(env, "cluster") == 0;
  if (force_streamk) return 0;
  int64_t max_len = 0, rows = 0;
  for (int b = 0; b < c->batch; ++b) {
    max_len = std::max<int64_t>(max_len, plen[b] + c->window);
    rows += (plen[b] + c->window) * c->num_heads;
  }
  int C = (int)std::min<int64_t>(16, std::max<int64_t>(2, (max_len + 63) / 64));
  // RSWA_DECODE_CLUSTER=2..16 sets the cluster size (for measurements)
  const char *cenv = getenv("RSWA_DECODE_CLUSTER");
  if (cenv) {
    const int c = atoi(cenv);
    if (c >= 2 && c <= 16) C = c;
  }
  const int64_t rings = (int64_t)c->batch * c->num_heads;
  // a few long rings need more CTAs than 16 per ring: stream-K spreads them
  // over the whole GPU (the merge then costs little next to the stream)
  const int64_t streamk_grid =
      std::min<int64_t>((int64_t)num_sms * decode_ctas_per_sm(c->dtype, c->head_dim),
                        (rows + kMinRowsPerCta - 1) / kMinRowsPerCta);
  if (!force_cluster && rings * C * 2 < streamk_grid) return 0;
  for (; C >= 2; C /= 2) {
    const int fit = decode_max_clusters(c->dtype, c->head_dim, C);
    if (fit >= rings) break;
    if (!force_cluster) return 0;
  }
  return C >= 2 ? C : 0;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

rswa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return RSWA_OK;
  g_last_cuda_error = e;
  return RSWA_ECUDA;
}

}  // namespace

// ---------------------------------------------------------------------------
extern "C" {

size_t rswa_cache_bytes(const rswa_config *cfg, const int64_t *prefill_len) {
  if (!config_ok(cfg, prefill_len)) return 0;
  size_t slots = 0;
  for (int b = 0; b < cfg->batch; ++b) slots += (size_t)(prefill_len[b] + cfg->window);
  return slots * (size_t)cfg->num_heads * (size_t)cfg->head_dim * elem_size(cfg);
}

size_t rswa_workspace_bytes(const rswa_config *cfg, const int64_t *prefill_len) {
  if (!config_ok(cfg, prefill_len)) return 0;
  const int dev = current_device();
  if (dev < 0) return 0;
  const DecodePlan p = plan_decode(cfg, prefill_len, nullptr, sm_count(dev),
                                   decode_ctas_per_sm(cfg->dtype, cfg->head_dim));
  return layout_ws(cfg, prefill_len, p).total;
}

size_t rswa_pool_cache_bytes(const rswa_config *cfg, int64_t pool_slots) {
  if (!cfg || pool_slots < 1) return 0;
  std::vector<int64_t> one(1, 0);
  rswa_config c1 = *cfg;
  c1.batch = 1;
  if (!config_ok(&c1, one.data())) return 0;
  if ((int64_t)cfg->num_heads * pool_slots >= (int64_t(1) << 40)) return 0;
  return (size_t)pool_slots * (size_t)cfg->num_heads * (size_t)cfg->head_dim * elem_size(cfg);
}

rswa_status rswa_state_create(const rswa_config *cfg, const int64_t *prefill_len,
                              const int64_t *n_generated, void *const *k_cache,
                              void *const *v_cache, void *workspace, size_t workspace_size,
                              void *stream, rswa_state **out) {
  return rswa_state_create_pooled(cfg, prefill_len, n_generated, nullptr, 0, k_cache, v_cache,
                                  workspace, workspace_size, stream, out);
}

rswa_status rswa_state_create_pooled(const rswa_config *cfg, const int64_t *prefill_len,
                                     const int64_t *n_generated, const int64_t *slot_base,
                                     int64_t pool_slots, void *const *k_cache,
                                     void *const *v_cache, void *workspace, size_t workspace_size,
                                     void *stream, rswa_state **out) {
  if (!out) return RSWA_EINVAL;
  *out = nullptr;
  if (!config_ok(cfg, prefill_len) || !k_cache || !v_cache || !workspace) return RSWA_EINVAL;
  if (slot_base) {
    // every request's range inside the pool, no two ranges overlapping
    if (pool_slots < 1 || (int64_t)cfg->num_heads * pool_slots >= (int64_t(1) << 40))
      return RSWA_EINVAL;
    std::vector<std::pair<int64_t, int64_t>> r((size_t)cfg->batch);
    for (int b = 0; b < cfg->batch; ++b) {
      const int64_t e = slot_base[b] + prefill_len[b] + cfg->window;
      if (slot_base[b] < 0 || e > pool_slots) return RSWA_EINVAL;
      r[(size_t)b] = {slot_base[b], e};
    }
    std::sort(r.begin(), r.end());
    for (size_t i = 1; i < r.size(); ++i)
      if (r[i].first < r[i - 1].second) return RSWA_EINVAL;
  }
  if (((uintptr_t)workspace & 255u) != 0) return RSWA_EINVAL;
  for (int l = 0; l < cfg->num_layers; ++l)
    if (!k_cache[l] || !v_cache[l] || !aligned16(k_cache[l]) || !aligned16(v_cache[l]))
      return RSWA_EINVAL;
  if (n_generated)
    for (int b = 0; b < cfg->batch; ++b)
      if (n_generated[b] < 0) return RSWA_EINVAL;
  const int dev = current_device();
  if (dev < 0) return RSWA_ECUDA;

  rswa_state *s = new (std::nothrow) rswa_state();
  if (!s) return RSWA_ENOMEM;
  s->cfg = *cfg;
  if (s->cfg.scale == 0.f) s->cfg.scale = 1.0f / sqrtf((float)cfg->head_dim);
  s->plen.assign(prefill_len, prefill_len + cfg->batch);
  s->slot_base.assign((size_t)cfg->batch, 0);
  s->pool_slots = 0;
  for (int b = 0; b < cfg->batch; ++b) {
    s->slot_base[(size_t)b] = slot_base ? slot_base[b] : s->pool_slots;
    if (!slot_base) s->pool_slots += prefill_len[b] + cfg->window;
  }
  if (slot_base) s->pool_slots = pool_slots;
  s->k_cache.assign(k_cache, k_cache + cfg->num_layers);
  s->v_cache.assign(v_cache, v_cache + cfg->num_layers);
  s->layer_ready.assign((size_t)cfg->num_layers, n_generated ? 1 : 0);
  s->workspace = workspace;
  s->workspace_size = workspace_size;
  s->device = dev;
  s->num_sms = sm_count(dev);
  s->plan = plan_decode(cfg, prefill_len, s->slot_base.data(), s->num_sms,
                        decode_ctas_per_sm(cfg->dtype, cfg->head_dim));
  s->ws = layout_ws(cfg, prefill_len, s->plan);
  if (workspace_size < s->ws.total) {
    delete s;
    return RSWA_ENOMEM;
  }

  // host images of the tables
  const int B = cfg->batch;
  std::vector<uint8_t> img(s->ws.total, 0);
  auto at = [&](size_t off) { return img.data() + off; };
  int64_t *t = (int64_t *)at(s->ws.t);
  int32_t *pl = (int32_t *)at(s->ws.plen);
  int64_t *sb = (int64_t *)at(s->ws.slot_base);
  int64_t *tb = (int64_t *)at(s->ws.tok_base);
  int32_t *tl = (int32_t *)at(s->ws.tile_base);
  int32_t *tl64 = (int32_t *)at(s->ws.tile64_base);
  int max_plen = 0;
  for (int b = 0; b < B; ++b) {
    t[b] = n_generated ? n_generated[b] : 0;
    t[B + b] = t[b];  // reset copy
    pl[b] = (int32_t)prefill_len[b];
    sb[b] = s->slot_base[(size_t)b];
    tb[b + 1] = tb[b] + prefill_len[b];
    tl[b + 1] = tl[b] + (int32_t)((prefill_len[b] + kPrefillTile - 1) / kPrefillTile);
    tl64[b + 1] = tl64[b] + (int32_t)((prefill_len[b] + kSimtTile - 1) / kSimtTile);
    max_plen = std::max(max_plen, (int)prefill_len[b]);
  }
  const std::vector<int4> pf_blocks = plan_prefill_blocks(cfg, prefill_len, s->num_sms);
  memcpy(at(s->ws.pf_blocks), pf_blocks.data(), pf_blocks.size() * sizeof(int4));
  memcpy(at(s->ws.pieces), s->plan.pieces.data(), s->plan.pieces.size() * sizeof(DecodePiece));
  memcpy(at(s->ws.cta_piece), s->plan.cta_piece.data(), s->plan.cta_piece.size() * sizeof(int32_t));
  memcpy(at(s->ws.bh_piece), s->plan.bh_piece.data(), s->plan.bh_piece.size() * sizeof(int32_t));
  // upload everything up to the partials (which the kernels overwrite)
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(workspace, img.data(), s->ws.part_ml, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    delete s;
    return from_cuda(e);
  }

  uint8_t *w = (uint8_t *)workspace;
  DeviceView &v = s->dv;
  v.B = B;
  v.H = cfg->num_heads;
  v.D = cfg->head_dim;
  v.W = cfg->window;
  v.L = cfg->num_layers;
  v.dtype = cfg->dtype;
  v.scale = s->cfg.scale;
  v.err = (int *)(w + s->ws.err);
  v.fault = (const int *)(w + s->ws.err) + 1;
  v.t = (int64_t *)(w + s->ws.t);
  v.plen = (const int32_t *)(w + s->ws.plen);
  v.slot_base = (const int64_t *)(w + s->ws.slot_base);
  v.tok_base = (const int64_t *)(w + s->ws.tok_base);
  v.tile_base = (const int32_t *)(w + s->ws.tile_base);
  v.tile64_base = (const int32_t *)(w + s->ws.tile64_base);
  v.pf_blocks = (const int4 *)(w + s->ws.pf_blocks);
  v.n_pf_blocks = (int)pf_blocks.size();
  v.pieces = (const DecodePiece *)(w + s->ws.pieces);
  v.cta_piece = (const int32_t *)(w + s->ws.cta_piece);
  v.bh_piece = (const int32_t *)(w + s->ws.bh_piece);
  v.bh_count = (int *)(w + s->ws.bh_count);
  v.part_ml = (float2 *)(w + s->ws.part_ml);
  v.part_o = (float *)(w + s->ws.part_o);
  v.decode_grid = s->plan.grid;
  v.n_pieces = s->plan.n_pieces;
  v.cluster_size = choose_cluster_size(cfg, prefill_len, s->num_sms);
  v.swa = 0;
  v.key_lo = 0;
  v.key_hi = INT_MAX;  // the whole cache
  v.out_ml = nullptr;
  v.out_o = nullptr;
  v.rope = RSWA_ROPE_NONE;
  v.rope_theta = 10000.f;
  v.rope_cs = (float2 *)(w + s->ws.rope_cs);
  v.total_tokens = tb[B];
  v.total_tiles = tl[B];
  v.total_tiles64 = tl64[B];
  v.max_plen = max_plen;
  *out = s;
  return RSWA_OK;
}

rswa_status rswa_state_destroy(rswa_state *state) {
  if (!state) return RSWA_EINVAL;
  delete state;
  return RSWA_OK;
}

int64_t rswa_cache_offset(const rswa_state *s, int32_t b, int32_t h, int64_t slot) {
  if (!s || b < 0 || b >= s->cfg.batch || h < 0 || h >= s->cfg.num_heads) return -1;
  const int64_t P = s->plen[(size_t)b];
  if (slot < 0 || slot >= P + s->cfg.window) return -1;
  const int64_t base = s->slot_base[(size_t)b];
  return ((int64_t)s->cfg.num_heads * base + (int64_t)h * (P + s->cfg.window) + slot) *
         s->cfg.head_dim;
}

rswa_status rswa_prefill(rswa_state *s, int32_t layer, const void *q, const void *k,
                         const void *v, void *out, void *stream) {
  if (!s || layer < 0 || layer >= s->cfg.num_layers) return RSWA_EINVAL;
  if (s->dv.total_tokens > 0 && (!q || !k || !v || !out)) return RSWA_EINVAL;
  if (s->dv.total_tokens > 0 &&
      (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)))
    return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  void *kc = s->k_cache[(size_t)layer];
  void *vc = s->v_cache[(size_t)layer];
  const int64_t kc_rows = (int64_t)s->cfg.num_heads * s->pool_slots;
  // the tensor-core kernel stores the prompt K/V into the cache itself; the
  // CUDA-core kernel takes a separate cache-fill pass
  const bool fused_fill = s->cfg.dtype == RSWA_BF16 && s->cfg.head_dim == 128;
  cudaError_t e = fused_fill ? cudaSuccess : launch_cache_fill(s->dv, k, v, kc, vc, st);
  // RoPE: rotated k overwrites the cache's prompt slots, rotated q goes to
  // `out`; attention then reads q from `out` and k from the cache
  const bool rope = s->dv.rope != RSWA_ROPE_NONE;
  if (e == cudaSuccess && rope) e = launch_rope_prefill(s->dv, q, k, out, kc, st);
  const void *qa = rope ? (const void *)out : q;
  const void *kca = rope ? (const void *)kc : nullptr;
  if (e == cudaSuccess) {
    if (fused_fill)
      e = launch_prefill_tc(s->dv, qa, k, v, out, s->dv.pf_blocks, s->dv.n_pf_blocks, kc, vc,
                            rope ? 1 : 0, kc_rows, st);
    else
      e = launch_prefill_simt(s->dv, qa, k, v, out, kca, st);
  }
  if (e != cudaSuccess) return from_cuda(e);
  s->layer_ready[(size_t)layer] = 1;
  return RSWA_OK;
}

rswa_status rswa_decode_step(rswa_state *s, int32_t layer, const void *q, const void *k_new,
                             const void *v_new, void *out, void *stream) {
  if (!s || layer < 0 || layer >= s->cfg.num_layers) return RSWA_EINVAL;
  if (!q || !k_new || !v_new || !out) return RSWA_EINVAL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out))
    return RSWA_EINVAL;
  if (!s->layer_ready[(size_t)layer]) return RSWA_ESTATE;
  if (current_device() != s->device) return RSWA_EINVAL;
  return from_cuda(launch_decode(s->dv, q, k_new, v_new, s->k_cache[(size_t)layer],
                                 s->v_cache[(size_t)layer], out, (cudaStream_t)stream, true));
}

rswa_status rswa_decode_step_partial(rswa_state *s, int32_t layer, const void *q,
                                     const void *k_new, const void *v_new, int64_t key_lo,
                                     int64_t key_hi, float *part_ml, float *part_o,
                                     void *stream) {
  if (!s || layer < 0 || layer >= s->cfg.num_layers) return RSWA_EINVAL;
  if (!q || !k_new || !v_new || !part_ml || !part_o) return RSWA_EINVAL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(part_ml) ||
      !aligned16(part_o))
    return RSWA_EINVAL;
  if (key_lo < 0 || key_hi < key_lo) return RSWA_EINVAL;
  if (!s->layer_ready[(size_t)layer]) return RSWA_ESTATE;
  if (current_device() != s->device) return RSWA_EINVAL;
  DeviceView v = s->dv;
  v.key_lo = (int)std::min<int64_t>(key_lo, INT_MAX);
  v.key_hi = (int)std::min<int64_t>(key_hi, INT_MAX);
  v.out_ml = reinterpret_cast<float2 *>(part_ml);
  v.out_o = part_o;
  return from_cuda(launch_decode(v, q, k_new, v_new, s->k_cache[(size_t)layer],
                                 s->v_cache[(size_t)layer], nullptr, (cudaStream_t)stream, true));
}

rswa_status rswa_combine_partials(const float *part_ml, const float *part_o, int32_t shares,
                                  int64_t rings, int32_t head_dim, int32_t dtype, void *out,
                                  void *stream) {
  if (shares < 1 || rings < 0 || (head_dim != 64 && head_dim != 128)) return RSWA_EINVAL;
  if (dtype != RSWA_F32 && dtype != RSWA_BF16) return RSWA_EINVAL;
  if (rings == 0) return RSWA_OK;
  if (!part_ml || !part_o || !out) return RSWA_EINVAL;
  return from_cuda(launch_combine(reinterpret_cast<const float2 *>(part_ml), part_o, shares, rings,
                                  head_dim, dtype, out, (cudaStream_t)stream));
}

rswa_status rswa_advance(rswa_state *s, void *stream) {
  if (!s) return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  return from_cuda(launch_advance(s->dv, (cudaStream_t)stream));
}

rswa_status rswa_reset_ring(rswa_state *s, void *stream) {
  if (!s) return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  cudaError_t e = cudaMemcpyAsync(s->dv.t, s->dv.t + s->cfg.batch,
                                  (size_t)s->cfg.batch * sizeof(int64_t),
                                  cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_rope_table(s->dv, (cudaStream_t)stream);
  return from_cuda(e);
}

rswa_status rswa_ngram_mask(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                            const int32_t *hist_len, int32_t rows, int32_t vocab, int32_t n,
                            int32_t window, int32_t *device_error, void *stream) {
  if (rows < 0 || vocab < 1 || n < 1 || window < 0 || ld < vocab || hist_ld < window)
    return RSWA_EINVAL;
  if (rows > 0 && (!logits || (window > 0 && !history))) return RSWA_EINVAL;
  if (rows == 0) return RSWA_OK;
  return from_cuda(launch_ngram(logits, ld, history, hist_ld, hist_len, rows, vocab, n, window,
                                device_error, (cudaStream_t)stream));
}

rswa_status rswa_ngram_topk(float *logits, int64_t ld, const int32_t *history, int64_t hist_ld,
                            const int32_t *hist_len, int32_t rows, int32_t vocab, int32_t n,
                            int32_t window, int32_t k, int32_t mask_in_place,
                            const float *uniform, float temperature, int32_t *top_idx,
                            float *top_val, int32_t *token, int32_t *device_error, void *stream) {
  static_assert(RSWA_TOPK_MAX == kTopkMax && RSWA_TOPK_MAX_VOCAB == kTopkMaxVocab,
                "header limits match the kernel");
  if (rows < 0 || vocab < 1 || vocab > kTopkMaxVocab || n < 1 || window < 0) return RSWA_EINVAL;
  if (k < 1 || k > kTopkMax || k > vocab) return RSWA_EINVAL;
  if (ld < vocab || (ld & 3) != 0 || hist_ld < window || window > kTopkMaxWindow)
    return RSWA_EINVAL;
  if (uniform && !(temperature > 0.f && isfinite(temperature))) return RSWA_EINVAL;
  if (rows == 0) return RSWA_OK;
  if (!logits || !aligned16(logits) || !top_idx || (window > 0 && !history)) return RSWA_EINVAL;
  return from_cuda(launch_ngram_topk(logits, ld, history, hist_ld, hist_len, rows, vocab, n,
                                     window, k, mask_in_place, uniform,
                                     uniform ? temperature : 1.f, top_idx, top_val, token,
                                     device_error, (cudaStream_t)stream));
}

rswa_status rswa_get_ring(const rswa_state *s, int64_t *n_generated, int32_t *ring_pos,
                          int64_t *cache_len, void *stream) {
  if (!s) return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  std::vector<int64_t> t((size_t)s->cfg.batch);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess)
    e = cudaMemcpy(t.data(), s->dv.t, t.size() * sizeof(int64_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return RSWA_ECUDA;
  const int64_t W = s->cfg.window;
  for (int b = 0; b < s->cfg.batch; ++b) {
    if (n_generated) n_generated[b] = t[(size_t)b];
    if (ring_pos) ring_pos[b] = (int32_t)(t[(size_t)b] < W ? 0 : t[(size_t)b] % W);
    if (cache_len) cache_len[b] = s->plen[(size_t)b] + std::min(t[(size_t)b], W);
  }
  return RSWA_OK;
}

rswa_status rswa_state_set_rope(rswa_state *s, int32_t policy, float theta, void *stream) {
  if (!s) return RSWA_EINVAL;
  if (policy != RSWA_ROPE_NONE && policy != RSWA_ROPE_ABSOLUTE && policy != RSWA_ROPE_SLOT)
    return RSWA_EINVAL;
  if (!(theta > 0.f) || !isfinite(theta)) return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  s->dv.rope = policy;
  s->dv.rope_theta = theta;
  return from_cuda(launch_rope_table(s->dv, (cudaStream_t)stream));
}

rswa_status rswa_state_set_attention(rswa_state *s, int32_t mode) {
  if (!s) return RSWA_EINVAL;
  if (mode != RSWA_ATTN_RING && mode != RSWA_ATTN_STANDARD_SWA) return RSWA_EINVAL;
  const bool swa = mode == RSWA_ATTN_STANDARD_SWA;
  if (swa != (s->dv.swa != 0)) {
    // re-plan the prefill blocks: one query tile per block with the window
    if (current_device() != s->device) return RSWA_EINVAL;
    const std::vector<int4> pf = plan_prefill_blocks(&s->cfg, s->plen.data(), s->num_sms, swa);
    cudaError_t e = cudaMemcpy((void *)s->dv.pf_blocks, pf.data(), pf.size() * sizeof(int4),
                               cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return from_cuda(e);
    s->dv.n_pf_blocks = (int)pf.size();
  }
  s->dv.swa = swa;
  // the window holds at most W keys per ring: one cluster of ceil(W / 64)
  // CTAs per ring (clusters are independent, so any batch size runs)
  const char *env = getenv("RSWA_DECODE_SPLIT");
  const bool force_streamk = env && strcmp(env, "streamk") == 0;
  if (s->dv.swa && !force_streamk)
    s->dv.cluster_size = std::max(1, std::min(16, (s->cfg.window + 63) / 64));
  else
    s->dv.cluster_size = choose_cluster_size(&s->cfg, s->plen.data(), s->num_sms);
  return RSWA_OK;
}

rswa_status rswa_decode_launch_shape(const rswa_state *s, int32_t *grid, int32_t *cluster_size) {
  if (!s) return RSWA_EINVAL;
  const int C = s->dv.cluster_size;
  if (grid) *grid = C > 0 ? s->cfg.batch * s->cfg.num_heads * C : s->dv.decode_grid;
  if (cluster_size) *cluster_size = C;
  return RSWA_OK;
}

rswa_status rswa_check_device_error(rswa_state *s, void *stream) {
  if (!s) return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  int word = 0;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&word, s->dv.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(s->dv.err, 0, sizeof(int));
  if (e != cudaSuccess) return RSWA_ECUDA;
  if (word & RSWA_DEVERR_TIMEOUT) return RSWA_ETIMEOUT;
  if (word) return RSWA_EDEVICE;
  return RSWA_OK;
}

int64_t rswa_debug_prefill_plan(const rswa_config *cfg, const int64_t *prefill_len,
                                int32_t num_sms, int32_t *out, int64_t capacity) {
  if (!config_ok(cfg, prefill_len) || num_sms < 1 || capacity < 0 || (capacity > 0 && !out))
    return -1;
  const std::vector<int4> blocks = plan_prefill_blocks(cfg, prefill_len, num_sms);
  const int64_t n = (int64_t)blocks.size();
  for (int64_t i = 0; i < n && i < capacity; ++i) {
    out[4 * i] = blocks[(size_t)i].x;
    out[4 * i + 1] = blocks[(size_t)i].y;
    out[4 * i + 2] = blocks[(size_t)i].z;
    out[4 * i + 3] = blocks[(size_t)i].w;
  }
  return n;
}

rswa_status rswa_debug_inject_fault(rswa_state *s, int32_t flags, void *stream) {
  if (!s || (flags & ~(RSWA_FAULT_DROP_DECODE_COPIES | RSWA_FAULT_DROP_PREFILL_LOADS)) != 0)
    return RSWA_EINVAL;
  if (current_device() != s->device) return RSWA_EINVAL;
  // the host value is staged by the copy before the call returns
  return from_cuda(cudaMemcpyAsync((int *)s->dv.fault, &flags, sizeof(int32_t),
                                   cudaMemcpyHostToDevice, (cudaStream_t)stream));
}

const char *rswa_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char *rswa_status_string(rswa_status st) {
  switch (st) {
    case RSWA_OK: return "ok";
    case RSWA_EINVAL: return "invalid argument";
    case RSWA_ENOMEM: return "workspace too small";
    case RSWA_ECUDA: return "CUDA call or kernel launch failed";
    case RSWA_ESTATE: return "call out of order (layer not prefilled)";
    case RSWA_ETIMEOUT: return "a kernel's bounded wait ran out";
    case RSWA_EDEVICE: return "a kernel rejected its data";
  }
  return "unknown status";
}

}  // extern "C"
