// R-SWA decode step: fused ring-slot write + split-K attention over the
// whole cache, then a log-sum-exp combine of the split partials.
//
// Method ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.1): each
// generated token's K/V goes to slot prefill_len + ring_pos (an append during
// warm-up, an overwrite once the cache holds prefill_len + W entries), and the
// token then attends to every entry of the cache.
//
// Design (HBM-bound: every cached K/V byte is read once per step):
//  - Work is split "stream-K" style: the flattened key rows of all (b, h)
//    rings are cut into equal contiguous ranges, one per CTA, so every CTA
//    streams the same number of bytes whatever the batch's raggedness.  A
//    CTA's range is a list of pieces, one per (b, h) ring it touches.
//  - One producer lane streams K and V rows into a 4-stage shared-memory ring
//    with bulk copies (cp.async.bulk, the TMA engine) completing on mbarriers;
//    four consumer warps compute.  The producer runs ahead across piece
//    boundaries so the copy pipeline never drains inside a CTA.
//  - Each row is handled by 8 lanes (16-byte chunks interleaved so a quarter
//    warp reads 128 contiguous bytes: no bank conflicts); the dot product is a
//    3-step xor-shuffle; softmax runs online in the log2 domain (exp2f).
//  - The CTA whose piece holds this step's write slot stores k_new/v_new to
//    the cache and substitutes them for that row from shared memory, so no CTA
//    ever uses the stale slot and nobody re-reads the fresh one.
//  - Each piece ends in an unnormalised partial (m, l, o[d]) in the
//    workspace.  The CTA that finishes the last piece of a (b, h) (a counter
//    per (b, h), bumped after a release fence) merges that ring's partials by
//    log-sum-exp and writes the output, then re-arms the counter: the combine
//    pass runs inside the same launch, overlapped with other CTAs' streaming.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"

namespace rswa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMergeBatch = 16;  // partials whose loads are in flight together in the merge
constexpr int kMaxCluster = 16;  // CTAs per ring in the cluster variant

template <typename T, int D>
struct DecodeShape {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kStageRows = 8192 / kRowBytes;  // 8 KB of K (and of V) per stage
  static constexpr int kStages = 4;
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;
  static constexpr int kGroups = kConsumerWarps * 4;  // 8 lanes per row
  static constexpr int kPasses = kStageRows / kGroups;
  static constexpr int kChunks = kRowBytes / 16;
  static constexpr int kChunksPerLane = kChunks / 8;
  static constexpr int kElemPerChunk = 16 / (int)sizeof(T);
  static constexpr int kEPL = kChunksPerLane * kElemPerChunk;  // elements per lane
  static_assert(kStageRows % kGroups == 0, "stage rows must split over the groups");
  static_assert(kChunks % 8 == 0, "row must be a multiple of 8 chunks");
  static_assert(kEPL * 8 == D, "lane split must cover the row");
};

// Stages of the shared-memory ring.  The cluster form serves short key
// ranges (a ring split 16 ways): three stages hold a CTA's whole range, and
// the smaller footprint lets three CTAs share an SM, so the next layer's
// CTAs become resident -- and request their prompt rows -- while this
// layer's are still running.
template <typename T, int D, bool kCluster>
constexpr int decode_stages() {
  return kCluster ? 3 : DecodeShape<T, D>::kStages;
}

template <typename T, int D, bool kCluster>
struct __align__(128) DecodeSmem {
  using S = DecodeShape<T, D>;
  static constexpr int NST = decode_stages<T, D, kCluster>();
  uint8_t k[NST][S::kStageRows * S::kRowBytes];
  uint8_t v[NST][S::kStageRows * S::kRowBytes];
  uint8_t sub_k[S::kRowBytes];
  uint8_t sub_v[S::kRowBytes];
  float red_o[S::kGroups][D];
  float red_m[S::kGroups];
  float red_l[S::kGroups];
  int is_last;
  // cluster variant: partials of the cluster's CTAs, written into the
  // leader's copy through distributed shared memory
  float cl_o[kCluster ? kMaxCluster : 1][D];
  float2 cl_ml[kCluster ? kMaxCluster : 1];
  uint64_t full[NST];
  uint64_t empty[NST];
};

// Rotate this lane's slice of a row (rotate-half RoPE, pairs (i, i + D/2))
// by the (cos, sin) table cs[D/2].  Lane li of a row's 8 lanes holds chunks
// li + 8 j; when a lane holds at least two chunks the partner chunk is in the
// same lane, otherwise (bf16, D = 64) it is in lane li ^ 4.
template <typename T, int D>
__device__ __forceinline__ void rope_lane(float *x, int li, const float2 *cs) {
  using S = DecodeShape<T, D>;
  constexpr int E = S::kElemPerChunk;
  if constexpr (S::kChunksPerLane >= 2) {
    constexpr int kHalf = S::kChunksPerLane / 2;
#pragma unroll
    for (int j = 0; j < kHalf; ++j)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float2 r = cs[(li + 8 * j) * E + e];
        const float a0 = x[j * E + e], b0 = x[(j + kHalf) * E + e];
        x[j * E + e] = a0 * r.x - b0 * r.y;
        x[(j + kHalf) * E + e] = b0 * r.x + a0 * r.y;
      }
  } else {
    const bool first = li < 4;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, x[e], 4);
      const float2 r = cs[(li & 3) * E + e];
      x[e] = first ? x[e] * r.x - other * r.y : x[e] * r.x + other * r.y;
    }
  }
}

// This step's key range of a piece, read after the grid-dependency wait:
// [kb, ke) clipped to the cache entries held (P_b + min(t_b + 1, W)), for the
// standard sliding window to the slots of the last W positions,
// [max(0, min(P_b, P_b + t_b - W + 1)), held), and to the caller's slot range
// [key_lo, key_hi) of a partial step.  A cluster CTA (rank of C) re-splits
// that window evenly.  wslot: this step's ring slot, or -1 when the piece
// lies wholly in the prompt (full ring mode only).
struct KeyRange {
  int kb, ke, wslot;
};
__device__ __forceinline__ KeyRange resolve_range(const DeviceView &v, const DecodePiece &pc,
                                                  int rank, int C) {
  KeyRange r{pc.key_begin, pc.key_end, -1};
  const bool windowed = v.swa || v.key_lo > 0 || v.key_hi < pc.plen + v.W;
  if (!windowed && r.ke <= pc.plen) return r;  // no ring counter needed
  const int64_t t = v.t[pc.b];
  int hi = pc.plen + (int)(t + 1 < (int64_t)v.W ? t + 1 : (int64_t)v.W);  // entries held
  r.wslot = pc.plen + (int)(t % v.W);
  if (windowed) {
    int lo = 0;
    if (v.swa) {
      const int64_t lo64 = (int64_t)pc.plen + t - v.W + 1;
      lo = lo64 < 0 ? 0 : (lo64 > pc.plen ? pc.plen : (int)lo64);
    }
    lo = max(lo, v.key_lo);  // the caller's key range (a share of a split cache)
    hi = min(hi, v.key_hi);
    if (lo > hi) lo = hi;
    if (C > 0) {
      const int per = (hi - lo + C - 1) / C;
      r.kb = min(lo + rank * per, hi);
      r.ke = min(lo + (rank + 1) * per, hi);
    } else {
      r.kb = max(r.kb, lo);
    }
  }
  r.ke = min(r.ke, hi);
  return r;
}

struct DecodeArgs {
  DeviceView v;
  const void *q, *k_new, *v_new;
  void *kc, *vc;
  void *out;
};


// Element tid of ring bh's result: the normalised output, or, for a partial
// step, the unnormalised (m, l, o) the caller combines with other shares.
template <typename T, int D>
__device__ __forceinline__ void store_result(const DeviceView &v, const DecodeArgs &a, int bh,
                                             int tid, float m, float l, float acc) {
  if (v.out_ml) {
    v.out_o[(int64_t)bh * D + tid] = acc;
    if (tid == 0) v.out_ml[bh] = make_float2(m, l);
  } else {
    ((T *)a.out)[(int64_t)bh * D + tid] = from_float<T>(acc / l);
  }
}

// kCluster = false: stream-K pieces from the work tables, partials merged
//   through global memory by the CTA that finishes a ring last.
// kCluster = true: one ring per cluster of v.cluster_size CTAs, each taking an
//   equal key range; partials go to the leader CTA's shared memory and one
//   cluster barrier replaces the global publish/merge (small batches, where
//   that hand-off dominates the step).
template <typename T, int D, bool kCluster>
__global__ void __launch_bounds__(DecodeShape<T, D>::kThreads)
    decode_split_kernel(const DecodeArgs a) {
  using S = DecodeShape<T, D>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem<T, D, kCluster> &sm = *reinterpret_cast<DecodeSmem<T, D, kCluster> *>(smem_raw);
  constexpr int NST = decode_stages<T, D, kCluster>();
  const DeviceView &v = a.v;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int p_begin = 0, p_end = 1, rank = 0;
  // The work plan is written once when the state is built, so this CTA's
  // first piece can be fetched before the grid-dependency wait below.
  DecodePiece first_piece;
  if constexpr (kCluster) {
    const int C = v.cluster_size;
    rank = (int)(blockIdx.x % (unsigned)C);
    const int ring = (int)(blockIdx.x / (unsigned)C);
    const int b = ring / v.H, h = ring % v.H;
    const int P = v.plen[b];
    const int len = P + v.W;
    const int per = (len + C - 1) / C;
    first_piece.row0 = (int64_t)v.H * v.slot_base[b] + (int64_t)h * len;
    first_piece.b = b;
    first_piece.h = h;
    first_piece.key_begin = min(rank * per, len);
    first_piece.key_end = min((rank + 1) * per, len);
    first_piece.plen = P;
    first_piece.first = 0;
    first_piece.count = C;
    first_piece.cta = (int)blockIdx.x;
  } else {
    p_begin = v.cta_piece[blockIdx.x];
    p_end = v.cta_piece[blockIdx.x + 1];
    first_piece = v.pieces[p_begin];
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], S::kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // Cluster variant: every thread arrives once at the start; consumers wait
  // on that phase before their first distributed-shared-memory store, so no
  // CTA writes into a peer that has not started.  (The producer warp arrives
  // and later exits; a cluster barrier waits only for non-exited threads.)
  if constexpr (kCluster) cluster_arrive_relaxed();

  // Prompt rows (slots < P_b) are written only by the prefill's cache fill
  // or by the caller, never by a kernel that lets its dependents start early
  // (only this kernel and the ring advance do, and neither writes a prompt
  // row).  So the first stages of this CTA's first piece that lie wholly in
  // the prompt can be requested before the grid-dependency wait; this
  // overlaps their memory latency with the tail of the previous layer.
  int pre_stages = 0;
  // Test-only fault injection: with RSWA_FAULT_DROP_DECODE_COPIES set the
  // producer issues no copy at all, so every consumer wait runs out, records
  // RSWA_DEVERR_TIMEOUT and the kernel still finishes.  The flag is written by
  // a host copy, which a kernel launched after it never overlaps.
  const bool drop_copies = (*v.fault & RSWA_FAULT_DROP_DECODE_COPIES) != 0;
  // (The standard-sliding-window mode picks its keys from t_b and a partial
  // step clips them to a slot range: no prefetch in either.)
  const bool prefetch_ok = !v.swa && v.key_lo == 0 && v.out_ml == nullptr;
  if (warp == S::kConsumerWarps && lane == 0 && !drop_copies && prefetch_ok) {
    const DecodePiece &pc = first_piece;
    const uint8_t *kbase = (const uint8_t *)a.kc + pc.row0 * S::kRowBytes;
    const uint8_t *vbase = (const uint8_t *)a.vc + pc.row0 * S::kRowBytes;
    for (int k0 = pc.key_begin; k0 < pc.key_end && pre_stages < NST;
         k0 += S::kStageRows) {
      const int rows = (pc.key_end - k0) < S::kStageRows ? (pc.key_end - k0) : S::kStageRows;
      if (k0 + rows > pc.plen) break;
      const uint32_t bytes = (uint32_t)rows * S::kRowBytes;
      mbar_arrive_expect_tx(&sm.full[pre_stages], 2 * bytes);
      bulk_g2s(sm.k[pre_stages], kbase + (int64_t)k0 * S::kRowBytes, bytes, &sm.full[pre_stages]);
      bulk_g2s(sm.v[pre_stages], vbase + (int64_t)k0 * S::kRowBytes, bytes, &sm.full[pre_stages]);
      ++pre_stages;
    }
  }
  // The first piece's q, k_new and v_new rows and its ring counter are read
  // right after the wait: start their trip to L2 now (a prefetch returns no
  // value, so a row still being written by an earlier kernel is read fresh).
  if (warp == 0 && lane < 7) {
    const int64_t in_off = ((int64_t)first_piece.b * v.H + first_piece.h) * D;
    const uint8_t *row = lane < 2 ? (const uint8_t *)a.q
                       : lane < 4 ? (const uint8_t *)a.k_new : (const uint8_t *)a.v_new;
    if (lane < 6)
      prefetch_l2(row + in_off * (int64_t)sizeof(T) + (lane & 1) * (D * sizeof(T) / 2));
    else
      prefetch_l2(v.t + first_piece.b);
  }
  // From here on the kernel reads q/k_new/v_new, the ring counters and ring
  // rows of the cache, which earlier kernels in the stream may still be
  // producing.
  grid_dependency_wait();
  allow_dependents();

  if (warp == S::kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0 || drop_copies) return;
    int stage = pre_stages % NST;
    uint32_t round = pre_stages / NST;
    bool dead = false;
    for (int p = p_begin; p < p_end && !dead; ++p) {
      const DecodePiece pc = p == p_begin ? first_piece : v.pieces[p];
      const KeyRange kr = resolve_range(v, pc, rank, kCluster ? v.cluster_size : 0);
      const int ke = kr.ke;
      const uint8_t *kbase = (const uint8_t *)a.kc + pc.row0 * S::kRowBytes;
      const uint8_t *vbase = (const uint8_t *)a.vc + pc.row0 * S::kRowBytes;
      const int k_first = kr.kb + (p == p_begin ? pre_stages * S::kStageRows : 0);
      for (int k0 = k_first; k0 < ke; k0 += S::kStageRows) {
        const int rows = (ke - k0) < S::kStageRows ? (ke - k0) : S::kStageRows;
        if (!mbar_wait_bounded(&sm.empty[stage], (round & 1) ^ 1, v.err, RSWA_DEVERR_TIMEOUT)) {
          dead = true;
          break;
        }
        const uint32_t bytes = (uint32_t)rows * S::kRowBytes;
        mbar_arrive_expect_tx(&sm.full[stage], 2 * bytes);
        bulk_g2s(sm.k[stage], kbase + (int64_t)k0 * S::kRowBytes, bytes, &sm.full[stage]);
        bulk_g2s(sm.v[stage], vbase + (int64_t)k0 * S::kRowBytes, bytes, &sm.full[stage]);
        if (++stage == NST) {
          stage = 0;
          ++round;
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;  // 0..127
  const int g = warp * 4 + (lane >> 3);
  const int li = lane & 7;
  int stage = 0;
  uint32_t round = 0;
  bool dead = false;

  for (int p = p_begin; p < p_end; ++p) {
    const DecodePiece pc = p == p_begin ? first_piece : v.pieces[p];
    const KeyRange kr = resolve_range(v, pc, rank, kCluster ? v.cluster_size : 0);
    const int ke = kr.ke, wslot = kr.wslot;
    const bool owner = wslot >= kr.kb && wslot < kr.ke;
    const int64_t in_off = ((int64_t)pc.b * v.H + pc.h) * D;  // element offset into [B][H][D]

    // q slice of this lane (rotated at its position with RoPE on), pre-scaled
    // into the log2 domain
    float qf[S::kEPL];
    {
      const uint8_t *qrow = (const uint8_t *)a.q + in_off * (int64_t)sizeof(T);
#pragma unroll
      for (int j = 0; j < S::kChunksPerLane; ++j) {
        const uint4 u = *reinterpret_cast<const uint4 *>(qrow + (li + 8 * j) * 16);
        Chunk<T>::widen(u, qf + j * S::kElemPerChunk);
      }
      if (v.rope) rope_lane<T, D>(qf, li, v.rope_cs + (int64_t)pc.b * (D / 2));
      const float qs = v.scale * kLog2e;
#pragma unroll
      for (int e = 0; e < S::kEPL; ++e) qf[e] *= qs;
    }

    if (owner) {
      // ring write of this step + shared-memory copy for the substitution
      const uint8_t *kn = (const uint8_t *)a.k_new + in_off * (int64_t)sizeof(T);
      const uint8_t *vn = (const uint8_t *)a.v_new + in_off * (int64_t)sizeof(T);
      const int64_t wrow = pc.row0 + wslot;
      uint8_t *kdst = (uint8_t *)a.kc + wrow * S::kRowBytes;
      uint8_t *vdst = (uint8_t *)a.vc + wrow * S::kRowBytes;
      if (!v.rope) {
        for (int c = tid; c < 2 * S::kChunks; c += 128) {
          const bool isk = c < S::kChunks;
          const int cc = isk ? c : c - S::kChunks;
          const uint4 u = *reinterpret_cast<const uint4 *>((isk ? kn : vn) + cc * 16);
          *reinterpret_cast<uint4 *>((isk ? sm.sub_k : sm.sub_v) + cc * 16) = u;
          *reinterpret_cast<uint4 *>((isk ? kdst : vdst) + cc * 16) = u;
        }
      } else {
        // k_new turns by its position before it enters the ring: chunk c and
        // chunk c + kChunks/2 hold the pairs (i, i + d/2)
        constexpr int kHalf = S::kChunks / 2;
        const float2 *cs = v.rope_cs + (int64_t)pc.b * (D / 2);
        for (int c = tid; c < kHalf + S::kChunks; c += 128) {
          if (c < kHalf) {
            float x[S::kElemPerChunk], y[S::kElemPerChunk];
            Chunk<T>::widen(*reinterpret_cast<const uint4 *>(kn + c * 16), x);
            Chunk<T>::widen(*reinterpret_cast<const uint4 *>(kn + (c + kHalf) * 16), y);
#pragma unroll
            for (int e = 0; e < S::kElemPerChunk; ++e) {
              const float2 r = cs[c * S::kElemPerChunk + e];
              const float a0 = x[e], b0 = y[e];
              x[e] = a0 * r.x - b0 * r.y;
              y[e] = b0 * r.x + a0 * r.y;
            }
            const uint4 ux = Chunk<T>::narrow(x), uy = Chunk<T>::narrow(y);
            *reinterpret_cast<uint4 *>(sm.sub_k + c * 16) = ux;
            *reinterpret_cast<uint4 *>(sm.sub_k + (c + kHalf) * 16) = uy;
            *reinterpret_cast<uint4 *>(kdst + c * 16) = ux;
            *reinterpret_cast<uint4 *>(kdst + (c + kHalf) * 16) = uy;
          } else {
            const int cc = c - kHalf;
            const uint4 u = *reinterpret_cast<const uint4 *>(vn + cc * 16);
            *reinterpret_cast<uint4 *>(sm.sub_v + cc * 16) = u;
            *reinterpret_cast<uint4 *>(vdst + cc * 16) = u;
          }
        }
      }
      named_bar_sync(1, 128);
    }

    float m = -INFINITY, l = 0.f;
    float o[S::kEPL];
#pragma unroll
    for (int e = 0; e < S::kEPL; ++e) o[e] = 0.f;

    for (int k0 = kr.kb; k0 < ke; k0 += S::kStageRows) {
      const int rows = (ke - k0) < S::kStageRows ? (ke - k0) : S::kStageRows;
      if (!dead && !mbar_wait_bounded(&sm.full[stage], round & 1, v.err, RSWA_DEVERR_TIMEOUT))
        dead = true;
      if (!dead) {
        const uint8_t *ks = sm.k[stage];
        const uint8_t *vs = sm.v[stage];
        float sc[S::kPasses];
#pragma unroll
        for (int ps = 0; ps < S::kPasses; ++ps) {
          const int r = ps * S::kGroups + g;
          // four independent partial sums: a 16-deep FMA chain would be the
          // latency of every row
          float a4[4] = {0.f, 0.f, 0.f, 0.f};
          if (r < rows) {
            const uint8_t *krow = (owner && k0 + r == wslot) ? sm.sub_k : ks + r * S::kRowBytes;
#pragma unroll
            for (int j = 0; j < S::kChunksPerLane; ++j) {
              const uint4 u = *reinterpret_cast<const uint4 *>(krow + (li + 8 * j) * 16);
              float kf[S::kElemPerChunk];
              Chunk<T>::widen(u, kf);
#pragma unroll
              for (int e = 0; e < S::kElemPerChunk; ++e)
                a4[e & 3] = fmaf(qf[j * S::kElemPerChunk + e], kf[e], a4[e & 3]);
            }
          }
          float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          acc += __shfl_xor_sync(0xffffffffu, acc, 1);
          acc += __shfl_xor_sync(0xffffffffu, acc, 2);
          acc += __shfl_xor_sync(0xffffffffu, acc, 4);
          sc[ps] = r < rows ? acc : -INFINITY;
        }
        float m_new = m;
#pragma unroll
        for (int ps = 0; ps < S::kPasses; ++ps) m_new = fmaxf(m_new, sc[ps]);
        if (m_new != -INFINITY) {
          const float corr = exp2f(m - m_new);
          l *= corr;
#pragma unroll
          for (int e = 0; e < S::kEPL; ++e) o[e] *= corr;
#pragma unroll
          for (int ps = 0; ps < S::kPasses; ++ps) {
            const int r = ps * S::kGroups + g;
            if (r < rows) {
              const float pr = exp2f(sc[ps] - m_new);
              l += pr;
              const uint8_t *vrow = (owner && k0 + r == wslot) ? sm.sub_v : vs + r * S::kRowBytes;
#pragma unroll
              for (int j = 0; j < S::kChunksPerLane; ++j) {
                const uint4 u = *reinterpret_cast<const uint4 *>(vrow + (li + 8 * j) * 16);
                float vf[S::kElemPerChunk];
                Chunk<T>::widen(u, vf);
#pragma unroll
                for (int e = 0; e < S::kElemPerChunk; ++e)
                  o[j * S::kElemPerChunk + e] = fmaf(pr, vf[e], o[j * S::kElemPerChunk + e]);
              }
            }
          }
          m = m_new;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[stage]);
      if (++stage == NST) {
        stage = 0;
        ++round;
      }
    }

    // -------- piece end: merge the 16 group states into one partial
    if (li == 0) {
      sm.red_m[g] = m;
      sm.red_l[g] = l;
    }
#pragma unroll
    for (int j = 0; j < S::kChunksPerLane; ++j)
#pragma unroll
      for (int e = 0; e < S::kElemPerChunk; ++e)
        sm.red_o[g][(li + 8 * j) * S::kElemPerChunk + e] = o[j * S::kElemPerChunk + e];
    named_bar_sync(1, 128);
    float M = -INFINITY;
#pragma unroll
    for (int gg = 0; gg < S::kGroups; ++gg) M = fmaxf(M, sm.red_m[gg]);
    float acc_e = 0.f;  // this thread's output element (tid < D)
    if (tid < D && M != -INFINITY)
#pragma unroll
      for (int gg = 0; gg < S::kGroups; ++gg)
        acc_e = fmaf(sm.red_o[gg][tid], exp2f(sm.red_m[gg] - M), acc_e);
    float L = 0.f;
    if (tid == 0 && M != -INFINITY)
      for (int gg = 0; gg < S::kGroups; ++gg) L = fmaf(sm.red_l[gg], exp2f(sm.red_m[gg] - M), L);
    if constexpr (kCluster) {
      // -------- hand the partial to the leader CTA's shared memory, then one
      // cluster barrier (release/acquire) and the leader merges
      cluster_wait_acquire();  // the start-of-kernel phase
      if (tid < D) st_cluster_f32(map_to_rank(&sm.cl_o[rank][tid], 0), acc_e);
      if (tid == 0) st_cluster_f32x2(map_to_rank(&sm.cl_ml[rank], 0), M, L);
      cluster_arrive_release();
      cluster_wait_acquire();
      if (rank == 0 && tid < D) {
        // unrolled to the largest cluster, so all C partials' loads and
        // exponentials are in flight together (a loop to the run-time C was
        // two dependent chains of C shared-memory loads)
        const int C = v.cluster_size;
        float2 ml[kMaxCluster];
        float ov[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          ml[r] = r < C ? sm.cl_ml[r] : make_float2(-INFINITY, 0.f);
          ov[r] = r < C ? sm.cl_o[r][tid] : 0.f;
        }
        float mx[4] = {ml[0].x, ml[1].x, ml[2].x, ml[3].x};
#pragma unroll
        for (int r = 4; r < kMaxCluster; ++r) mx[r & 3] = fmaxf(mx[r & 3], ml[r].x);
        const float Mg = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        float Lg = 0.f, acc = 0.f;
        if (Mg != -INFINITY) {
          float l4[4] = {0.f, 0.f, 0.f, 0.f}, a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r) {
            const float wgt = exp2f(ml[r].x - Mg);  // 0 for an empty range or an absent rank
            l4[r & 3] = fmaf(wgt, ml[r].y, l4[r & 3]);
            a4[r & 3] = fmaf(wgt, ov[r], a4[r & 3]);
          }
          Lg = (l4[0] + l4[1]) + (l4[2] + l4[3]);
          acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        }
        store_result<T, D>(v, a, pc.b * v.H + pc.h, tid, Mg, Lg, acc);
      }
      continue;  // a cluster CTA has exactly one piece
    }
    if (tid < D) v.part_o[(int64_t)p * D + tid] = acc_e;
    if (tid == 0) v.part_ml[p] = make_float2(M, L);
    // -------- publish the partial; the last piece of this (b, h) merges.
    // The barrier orders every thread's partial stores before thread 0's
    // acq_rel atomic, whose release makes them visible device-wide and whose
    // acquire (in the last CTA) orders the merge's loads after all of them.
    named_bar_sync(1, 128);
    const int p0 = pc.first, np = pc.count;
    const int bh = pc.b * v.H + pc.h;
    if (tid == 0) {
      int last = 1;
      if (np > 1) {
        int old;
        asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;"
                     : "=r"(old)
                     : "l"(v.bh_count + bh)
                     : "memory");
        last = old == np - 1;
        if (last) v.bh_count[bh] = 0;  // re-arm for the next launch
      }
      sm.is_last = last;
    }
    named_bar_sync(1, 128);
    if (sm.is_last) {
      // Thread tid merges output element tid.  Partials are read straight
      // from L2, kMergeBatch at a time with every load of a batch in flight
      // together, merged online by log-sum-exp.
      float Mg = -INFINITY, Lg = 0.f, acc = 0.f;
      for (int c0 = 0; c0 < np; c0 += kMergeBatch) {
        float2 ml[kMergeBatch];
        float ov[kMergeBatch];
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
          const bool ok = c0 + i < np;
          const int64_t pp = p0 + c0 + i;
          ml[i] = ok ? __ldcg(&v.part_ml[pp]) : make_float2(-INFINITY, 0.f);
          ov[i] = (ok && tid < D) ? __ldcg(&v.part_o[pp * D + tid]) : 0.f;
        }
        float Mc = Mg;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) Mc = fmaxf(Mc, ml[i].x);
        if (Mc == -INFINITY) continue;
        const float corr = exp2f(Mg - Mc);
        Lg *= corr;
        acc *= corr;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
          const float wgt = exp2f(ml[i].x - Mc);  // 0 for empty or absent pieces
          Lg = fmaf(wgt, ml[i].y, Lg);
          acc = fmaf(wgt, ov[i], acc);
        }
        Mg = Mc;
      }
      if (tid < D) store_result<T, D>(v, a, bh, tid, Mg, Lg, acc);
    }
  }
}

__global__ void advance_kernel(int64_t *t, int B) {
  grid_dependency_wait();  // the decode kernels before it read t
  allow_dependents();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) t[b] += 1;
}

template <typename T, int D, bool kCluster>
cudaError_t set_smem_attr() {
  const int smem = (int)sizeof(DecodeSmem<T, D, kCluster>);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<T, D, kCluster>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess && kCluster)
    e = cudaFuncSetAttribute(decode_split_kernel<T, D, kCluster>,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <typename T, int D, bool kCluster>
cudaError_t launch_decode_t(const DeviceView &v, const void *q, const void *k_new,
                            const void *v_new, void *kc, void *vc, void *out, cudaStream_t s,
                            bool pdl) {
  using S = DecodeShape<T, D>;
  static bool attr_set = false;  // per instantiation; also set when the state is built
  if (!attr_set) {
    cudaError_t e = set_smem_attr<T, D, kCluster>();
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  DecodeArgs a{v, q, k_new, v_new, kc, vc, out};
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(kCluster ? v.B * v.H * v.cluster_size : v.decode_grid);
  lc.blockDim = dim3(S::kThreads);
  lc.dynamicSmemBytes = sizeof(DecodeSmem<T, D, kCluster>);
  lc.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  int na = 1;
  if (kCluster) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)v.cluster_size;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    na = 2;
  }
  lc.attrs = attr;
  lc.numAttrs = na;
  return cudaLaunchKernelEx(&lc, decode_split_kernel<T, D, kCluster>, a);
}

template <typename T, int D>
cudaError_t launch_decode_d(const DeviceView &v, const void *q, const void *k_new,
                            const void *v_new, void *kc, void *vc, void *out, cudaStream_t s,
                            bool pdl) {
  return v.cluster_size > 0
             ? launch_decode_t<T, D, true>(v, q, k_new, v_new, kc, vc, out, s, pdl)
             : launch_decode_t<T, D, false>(v, q, k_new, v_new, kc, vc, out, s, pdl);
}

template <typename T, int D>
int ctas_per_sm_t() {
  using S = DecodeShape<T, D>;
  if (set_smem_attr<T, D, false>() != cudaSuccess) return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_split_kernel<T, D, false>,
                                                    S::kThreads,
                                                    sizeof(DecodeSmem<T, D, false>)) !=
          cudaSuccess ||
      n < 1)
    return 1;
  return n;
}

// Clusters of `cluster` CTAs that can be resident at once (0 if unsupported).
template <typename T, int D>
int max_clusters_t(int cluster) {
  using S = DecodeShape<T, D>;
  if (set_smem_attr<T, D, true>() != cudaSuccess) return 0;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(cluster * 1024);
  lc.blockDim = dim3(S::kThreads);
  lc.dynamicSmemBytes = sizeof(DecodeSmem<T, D, true>);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_split_kernel<T, D, true>, &lc) != cudaSuccess)
    return 0;
  return n;
}

}  // namespace

cudaError_t launch_decode(const DeviceView &v, const void *q, const void *k_new,
                          const void *v_new, void *kc, void *vc, void *out, cudaStream_t s,
                          bool pdl) {
  if (v.dtype == RSWA_BF16) {
    if (v.D == 128)
      return launch_decode_d<__nv_bfloat16, 128>(v, q, k_new, v_new, kc, vc, out, s, pdl);
    return launch_decode_d<__nv_bfloat16, 64>(v, q, k_new, v_new, kc, vc, out, s, pdl);
  }
  if (v.D == 128) return launch_decode_d<float, 128>(v, q, k_new, v_new, kc, vc, out, s, pdl);
  return launch_decode_d<float, 64>(v, q, k_new, v_new, kc, vc, out, s, pdl);
}

// Log-sum-exp merge of `shares` partials (m, l, o) per ring: one CTA per ring,
// one thread per output element.
template <typename T>
__global__ void combine_kernel(const float2 *__restrict__ ml, const float *__restrict__ o,
                               int shares, int64_t rings, int D, T *__restrict__ out) {
  const int64_t bh = blockIdx.x;
  const int e = threadIdx.x;
  float Mg = -INFINITY;
  for (int g = 0; g < shares; ++g) Mg = fmaxf(Mg, ml[(int64_t)g * rings + bh].x);
  float Lg = 0.f, acc = 0.f;
  if (Mg != -INFINITY)
    for (int g = 0; g < shares; ++g) {
      const float2 p = ml[(int64_t)g * rings + bh];
      const float wgt = exp2f(p.x - Mg);  // 0 for an empty share
      Lg = fmaf(wgt, p.y, Lg);
      acc = fmaf(wgt, o[((int64_t)g * rings + bh) * D + e], acc);
    }
  out[bh * D + e] = from_float<T>(acc / Lg);
}

cudaError_t launch_combine(const float2 *ml, const float *o, int shares, int64_t rings, int D,
                           int dtype, void *out, cudaStream_t s) {
  if (dtype == RSWA_BF16)
    combine_kernel<__nv_bfloat16><<<(unsigned)rings, D, 0, s>>>(ml, o, shares, rings, D,
                                                                (__nv_bfloat16 *)out);
  else
    combine_kernel<float><<<(unsigned)rings, D, 0, s>>>(ml, o, shares, rings, D, (float *)out);
  return cudaGetLastError();
}

cudaError_t launch_advance(const DeviceView &v, cudaStream_t s) {
  if (v.rope) return launch_advance_rope(v, s);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((v.B + 255) / 256);
  lc.blockDim = dim3(256);
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, advance_kernel, v.t, v.B);
}

int decode_max_clusters(int dtype, int head_dim, int cluster) {
  if (dtype == RSWA_BF16)
    return head_dim == 128 ? max_clusters_t<__nv_bfloat16, 128>(cluster)
                           : max_clusters_t<__nv_bfloat16, 64>(cluster);
  return head_dim == 128 ? max_clusters_t<float, 128>(cluster) : max_clusters_t<float, 64>(cluster);
}

int decode_ctas_per_sm(int dtype, int head_dim) {
  if (dtype == RSWA_BF16)
    return head_dim == 128 ? ctas_per_sm_t<__nv_bfloat16, 128>() : ctas_per_sm_t<__nv_bfloat16, 64>();
  return head_dim == 128 ? ctas_per_sm_t<float, 128>() : ctas_per_sm_t<float, 64>();
}

}  // namespace rswa
