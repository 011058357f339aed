// Prefill causal attention on the 5th-generation tensor cores (bf16, d = 128).
//
// Method ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.1): the
// prefill segment keeps full attention -- every prompt token attends causally
// to all earlier tokens of its prompt.  The page's section 三 notes that the
// transformers path materialises the whole score matrix; here it is a
// flash-style kernel that never leaves the chip with it.
//
// One CTA computes two consecutive 128-row query tiles A and B = A + 1 of one
// (sequence, head); both read every K/V tile they need once from shared
// memory:
//   warp 8      TMA producer: Q_A and Q_B once, then K tiles (128 keys x 128
//               dims, bf16, 128-byte swizzle) into a 2-stage ring;
//   warp 10     TMA producer of the V tiles (3-stage ring);
//   warp 9      MMA issuer (one thread) and TMEM owner (512 columns:
//               S_A, S_B, O_A, O_B, 128 fp32 columns each).  Order per key
//               tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so each softmax
//               warpgroup works while the tensor core runs the other tile's
//               MMAs.  P_X(j) overwrites S_X(j)'s columns as bf16 pairs and is
//               the A operand (from TMEM) of PV_X(j);
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: thread r of a
//               warpgroup owns query row r (TMEM lane r).  It loads its S row,
//               masks the diagonal tile, runs the online softmax in the log2
//               domain and writes P back to TMEM.  O is only rescaled when a
//               warp's running max grows by more than 2^8; otherwise the stale
//               max keeps every p <= 256, exact in the end because l uses the
//               same max.  The epilogue divides by l and stores bf16 rows.
// Warps 8-11 (warp 11 has no role) hand registers to the softmax warpgroups
// (setmaxnreg), which hold a whole 128-score row per thread.
// Blocks are grouped by (sequence, head), longest first inside a group, so
// the CTAs running together share their K/V tiles through L2.  Every mbarrier
// wait is bounded; on a timeout the kernel records it, stops issuing work,
// waits (bounded) for what is in flight, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tmap.h"

namespace rswa {
namespace {

constexpr int kTile = 128;   // query rows and keys per tile
constexpr int kD = 128;      // head dim
constexpr int kKStages = 2;  // K ring depth
constexpr int kVStages = 3;  // V ring depth: a V tile is held until PV_B is done, and a
                             // 32 KB tile load takes ~2.8 us under full load
constexpr int kHalfBytes = kTile * 64 * 2;   // one 64-column swizzled half: 16 KB
constexpr int kTileBytes = 2 * kHalfBytes;   // 32 KB
constexpr int kThreads = 384;       // three warpgroups: softmax A, softmax B, the rest
constexpr int kLaunchRegs = 168;    // registers per thread at launch (65,536 / 384, rounded down to 8)
// Registers per thread after the split: the softmax warpgroups hold a whole
// 128-score row in registers; the loader / MMA warpgroup needs few.
constexpr int kSoftmaxRegs = 224;
constexpr int kAuxRegs = 56;
static_assert(256 * kSoftmaxRegs + 128 * kAuxRegs <= kThreads * kLaunchRegs,
              "register split above the launch's registers");
constexpr int kProducerWarp = 8;   // Q and K loads
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10; // V loads
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// 1 in kEmuEvery exponential pairs uses the FMA-pipe exp2 (0: none, every
// exponential on MUFU).  Build-time knob: -DRSWA_EXP2_FMA_EVERY=N.
#ifndef RSWA_EXP2_FMA_EVERY
#define RSWA_EXP2_FMA_EVERY 0
#endif
constexpr int kEmuEvery = RSWA_EXP2_FMA_EVERY;
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr uint32_t col_s(int x) { return (uint32_t)x * kTile; }        // 0, 128
__host__ __device__ constexpr uint32_t col_o(int x) { return 256u + (uint32_t)x * kTile; } // 256, 384

struct __align__(1024) PrefillSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2];    // per query tile: S_X(j) finished
  uint64_t p_full[2];    // per query tile: P_X(j) written (4 warp arrivals)
  uint64_t o_final[2];   // per query tile: the last PV_X finished
  uint64_t mma_done;     // everything the MMA thread issued finished
  uint32_t tmem_base;
  int dead;
};

struct PrefillTcArgs {
  DeviceView v;
  const int4 *blocks;  // (b, h, first query tile, number of tiles 1|2)
  __nv_bfloat16 *out;
  __nv_bfloat16 *kc, *vc;  // this layer's caches (prompt rows of a ragged last tile)
  int k_from_cache;    // K tiles from the layer's cache (rotated keys) instead of k
  int store_k, store_v;  // store the block's own K / V tiles into the cache
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int *err,
                                         volatile int *dead) {
  if (*dead) return false;
  if (mbar_wait_bounded(bar, parity, err, RSWA_DEVERR_TIMEOUT)) return true;
  *dead = 1;
  return false;
}

// Issue the 8 K-steps of S = Q K^T (M = N = 128, K = 128 dims).
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = tc::idesc_bf16_f32(kTile, kTile, false, false);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const uint32_t off = (uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32;
    tc::mma_ss(d_tmem, tc::sw128_desc(q_addr + off, 16, 1024),
               tc::sw128_desc(k_addr + off, 16, 1024), idesc, kk > 0);
  }
}

// Issue the 8 K-steps of O (+)= P V (M = 128 rows, N = 128 dims, K = 128 keys).
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_addr,
                                         bool accumulate) {
  constexpr uint32_t idesc = tc::idesc_bf16_f32(kTile, kD, false, true);
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    tc::mma_ts(o_tmem, p_tmem + (uint32_t)kk * 8,
               tc::sw128_desc(v_addr + (uint32_t)kk * 2048, kHalfBytes, 1024), idesc,
               (accumulate || kk > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc, const PrefillTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // dynamic shared memory is only 16-byte aligned: round up to 1024 for the swizzle atoms
  PrefillSmem &sm = *reinterpret_cast<PrefillSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const DeviceView &v = a.v;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int4 blk = a.blocks[blockIdx.x];
  const int b = blk.x, h = blk.y, qt0 = blk.z, ntiles = blk.w;
  const int P = v.plen[b];
  const int tok0 = (int)v.tok_base[b];
  // Key tiles j0 .. qt of query tile qt: j0 = 0 (causal), or, for the
  // standard sliding window, the tile of the first key in the window of the
  // block's first query (blocks then hold one query tile).  Loops below count
  // iterations from 0; key tile = j0 + iteration.
  const int j0 = v.swa ? max(0, qt0 * kTile - v.W + 1) / kTile : 0;
  const int n_kv_a = qt0 + 1 - j0, n_kv_b = ntiles > 1 ? qt0 + 2 - j0 : 0;
  const int n_kv_all = qt0 + ntiles - j0;
  // The cache fill (prompt K/V into cache slots [0, P_b)) rides on the loads:
  // a block's last key tiles are its own query tiles qt0 .. qt0 + ntiles - 1
  // (the diagonal), which no other block owns, so every prompt tile is stored
  // exactly once.  They are the last loads of both rings, so their slots are
  // never refilled.  A whole tile goes out by TMA store from the shared-memory
  // tile the MMAs read; the rows of a ragged last tile (its rest would land
  // in ring slots) by plain stores in the epilogue.
  const int64_t crow0 = (int64_t)v.H * v.slot_base[b] + (int64_t)h * (P + v.W);
  const int n_full_tiles = P / kTile;  // tiles lying wholly in the prompt

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 4);
      mbar_init(&sm.o_final[x], 1);
    }
    mbar_init(&sm.mma_done, 1);
    sm.dead = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = sm.tmem_base;
  volatile int *dead = &sm.dead;

  // Registers move from the loader / MMA warpgroup (warps 8-11; warp 11 has
  // no role) to the two softmax warpgroups.  Each warpgroup changes its count
  // at the top of its own branch, so the compiler allocates each branch
  // within its own count.
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kAuxRegs));
    if (warp == kProducerWarp || warp == kVProducerWarp) {
      // ------------------------------------------------------------ producers
      // warp 8 loads Q and the K ring, warp 10 the V ring, so a K load never
      // waits behind a V slot that is still in use (and the other way round).
      if (lane == 0) {
        const bool is_k = warp == kProducerWarp;
        // test-only fault injection: no loads at all, so every wait on them
        // runs out (bounded) and the kernel takes its timeout path
        const bool drop_loads = (*v.fault & RSWA_FAULT_DROP_PREFILL_LOADS) != 0;
        const int xh = h * kD;
        const CUtensorMap *tm = is_k ? &tm_k : &tm_v;
        const int nst = is_k ? kKStages : kVStages;
        tc::prefetch_tmap(tm);
        if (is_k && !drop_loads) {
          tc::prefetch_tmap(&tm_q);
          mbar_arrive_expect_tx(&sm.q_full, (uint32_t)(ntiles * kTileBytes));
          for (int x = 0; x < ntiles; ++x) {
            const int y = tok0 + (qt0 + x) * kTile;
            tc::tma_load_2d(sm.q[x], &tm_q, xh, y, &sm.q_full);
            tc::tma_load_2d(sm.q[x] + kHalfBytes, &tm_q, xh + 64, y, &sm.q_full);
          }
        }
        int issued = 0;
        // K from the cache: rows H * S_b + h * (P_b + W) + key of a [rows][128]
        // map (rows past the prompt are ring slots: masked, like the causal
        // overhang of the input layout)
        const bool from_cache = is_k && a.k_from_cache;
        const int x0 = from_cache ? 0 : xh;
        const int y0 = from_cache ? (int)((int64_t)v.H * v.slot_base[b] + (int64_t)h * (P + v.W))
                                  : tok0;
        for (int j = 0; !drop_loads && j < n_kv_all; ++j) {
          const int s = j % nst;
          uint64_t *empty = is_k ? &sm.k_empty[s] : &sm.v_empty[s];
          uint64_t *full = is_k ? &sm.k_full[s] : &sm.v_full[s];
          uint8_t *dst = is_k ? sm.k[s] : sm.v[s];
          if (!wait_bar(empty, ((j / nst) & 1) ^ 1, v.err, dead)) break;
          mbar_arrive_expect_tx(full, kTileBytes);
          tc::tma_load_2d(dst, tm, x0, y0 + (j0 + j) * kTile, full);
          tc::tma_load_2d(dst + kHalfBytes, tm, x0 + 64, y0 + (j0 + j) * kTile, full);
          issued = j + 1;
        }
        // every load issued has landed before the CTA may exit (bounded)
        if (is_k && !drop_loads) mbar_wait_bounded(&sm.q_full, 0, v.err, RSWA_DEVERR_TIMEOUT);
        for (int s = 0; s < nst && s < issued; ++s) {
          const int last = s + ((issued - 1 - s) / nst) * nst;
          mbar_wait_bounded(is_k ? &sm.k_full[s] : &sm.v_full[s], (last / nst) & 1, v.err,
                            RSWA_DEVERR_TIMEOUT);
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t q_addr0 = smem_u32(sm.q[0]);
        // key tile j0 + it lands in K slot it mod 2 / V slot it mod 3; send it to
        // the cache if it is one of this block's whole prompt tiles
        bool stored = false;
        auto store_tile = [&](const CUtensorMap *tm, const uint8_t *src, int it) {
          const int kt = j0 + it;
          if (kt < qt0 || kt >= n_full_tiles) return;
          const int y = (int)(crow0 + (int64_t)kt * kTile);
          tc::tma_store_2d(tm, src, 0, y);
          tc::tma_store_2d(tm, src + kHalfBytes, 64, y);
          stored = true;
        };
        bool ok = wait_bar(&sm.q_full, 0, v.err, dead) &&
                  wait_bar(&sm.k_full[0], 0, v.err, dead);
        if (ok) {
          tc::fence_after_sync();
          if (a.store_k) store_tile(&tm_kc, sm.k[0], 0);
          for (int x = 0; x < ntiles; ++x) {
            issue_qk(tbase + col_s(x), q_addr0 + (uint32_t)x * kTileBytes, smem_u32(sm.k[0]));
            tc::commit(&sm.s_full[x]);
          }
          tc::commit(&sm.k_empty[0]);
        }
        for (int j = 0; ok && j < n_kv_all; ++j) {
          const int s = j % kVStages;          // V stage of tile j
          const int s1 = (j + 1) % kKStages;   // K stage of tile j + 1
          bool k1_ready = false;  // K_{j+1} waited for
          if (!(ok = wait_bar(&sm.v_full[s], (j / kVStages) & 1, v.err, dead))) break;
          if (a.store_v) store_tile(&tm_vc, sm.v[s], j);
          // K_{j+1} has usually landed by now: taking it here keeps the barrier
          // check out of the gap between P V and the next Q K^T of tile A (a
          // wait issued right after a burst of MMAs costs 50-200 cycles).  If
          // it has not, it is waited for there, as before.
          if (j + 1 < n_kv_all && mbar_try_wait(&sm.k_full[s1], ((j + 1) / kKStages) & 1)) {
            tc::fence_after_sync();
            k1_ready = true;
            if (a.store_k) store_tile(&tm_kc, sm.k[s1], j + 1);
          }
          for (int x = 0; x < ntiles; ++x) {
            const int nkv = x == 0 ? n_kv_a : n_kv_b;
            if (j >= nkv) continue;
            // O_X += P_X(j) V_j
            if (!(ok = wait_bar(&sm.p_full[x], j & 1, v.err, dead))) break;
            tc::fence_after_sync();
            issue_pv(tbase + col_o(x), tbase + col_s(x), smem_u32(sm.v[s]), j > 0);
            if (j == nkv - 1) tc::commit(&sm.o_final[x]);
            // S_X(j+1) = Q_X K_{j+1}^T  (overwrites P_X(j): issued after PV_X(j))
            if (j + 1 < nkv) {
              if (!k1_ready) {
                if (!(ok = wait_bar(&sm.k_full[s1], ((j + 1) / kKStages) & 1, v.err, dead))) break;
                tc::fence_after_sync();
                k1_ready = true;
                if (a.store_k) store_tile(&tm_kc, sm.k[s1], j + 1);
              }
              issue_qk(tbase + col_s(x), q_addr0 + (uint32_t)x * kTileBytes, smem_u32(sm.k[s1]));
              tc::commit(&sm.s_full[x]);
            }
          }
          if (!ok) break;
          tc::commit(&sm.v_empty[s]);
          if (k1_ready) tc::commit(&sm.k_empty[s1]);
        }
        tc::commit(&sm.mma_done);
        if (stored) {
          tc::store_commit();
          tc::store_wait_read();  // the tiles stay in shared memory until read
        }
        mbar_wait_bounded(&sm.mma_done, 0, v.err, RSWA_DEVERR_TIMEOUT);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------------------------------------------------------ softmax
    const int x = warp >> 2;          // query tile of this warpgroup (0 = A, 1 = B)
    const int wq = warp & 3;          // warp inside the warpgroup = TMEM lane quarter
    const int r = wq * 32 + lane;     // query row inside the tile
    const int qt = qt0 + x;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t t_s = tbase + lane_off + col_s(x);
    const uint32_t t_o = tbase + lane_off + col_o(x);
    const float sl2 = v.scale * kLog2e;
    float m_run = -INFINITY, l_run = 0.f;
    const int nkv = x == 0 ? n_kv_a : n_kv_b;
    bool ok = x < ntiles;
    for (int j = 0; ok && j < nkv; ++j) {
      ok = wait_bar(&sm.s_full[x], j & 1, v.err, dead);
      if (!ok) break;
      tc::fence_after_sync();
      float s[kTile];
      tc::ld32(t_s + 0, reinterpret_cast<uint32_t *>(s));
      tc::ld32(t_s + 32, reinterpret_cast<uint32_t *>(s) + 32);
      tc::ld32(t_s + 64, reinterpret_cast<uint32_t *>(s) + 64);
      tc::ld32(t_s + 96, reinterpret_cast<uint32_t *>(s) + 96);
      tc::wait_ld();
      if (j0 + j == qt) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c > r) s[c] = -INFINITY;
      }
      if (v.swa) {
        // keys before the window of query row r: key < query - W + 1
        const int lim = (qt - j0 - j) * kTile + r - v.W + 1;
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c < lim) s[c] = -INFINITY;
      }
      // row max as an 8-way tree (a single running max would be a 128-deep
      // dependency chain)
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int c = 8; c < kTile; c += 2) mx8[(c >> 1) & 7] = tc::fmax3(mx8[(c >> 1) & 7], s[c], s[c + 1]);
      float mx = tc::fmax3(tc::fmax3(mx8[0], mx8[1], mx8[2]), tc::fmax3(mx8[3], mx8[4], mx8[5]),
                           fmaxf(mx8[6], mx8[7]));
      mx *= sl2;
      const float m_new = fmaxf(m_run, mx);
      const bool need = j > 0 && m_new > m_run + kRescaleThreshold;
      const bool rescale = __any_sync(0xffffffffu, need);
      float m_use = m_run, alpha = 1.f;
      if (j == 0) {
        m_use = m_new;
      } else if (rescale) {
        m_use = m_new;
        alpha = tc::ex2(m_run - m_new);
      }
      uint64_t rs4[4];  // row sum as 4 packed pairs of partial sums
#pragma unroll
      for (int i = 0; i < 4; ++i) rs4[i] = 0;
      const uint64_t sl2x2 = tc::f2_pack(sl2, sl2);
      // a row whose keys so far are all outside its window has m = -inf:
      // its p are 0 (2^-inf), and the next tile's max rescales O and l by 0
      const float m_sub = m_use == -INFINITY ? 0.f : m_use;
      const uint64_t negm2 = tc::f2_pack(-m_sub, -m_sub);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          // x = s * scale*log2(e) - m for the pair, one packed FMA
          const uint64_t xx = tc::ffma2(tc::f2_pack(s[64 * half + 2 * c], s[64 * half + 2 * c + 1]),
                                        sl2x2, negm2);
          const float x0 = tc::f2_lo(xx), x1 = tc::f2_hi(xx);
          // one pair in kEmuEvery on the FMA pipe, the rest on MUFU
          const bool emu = kEmuEvery > 0 && (c % (kEmuEvery > 0 ? kEmuEvery : 1)) == kEmuEvery - 1;
          const float p0 = emu ? tc::exp2_fma(x0) : tc::ex2(x0);
          const float p1 = emu ? tc::exp2_fma(x1) : tc::ex2(x1);
          rs4[c & 3] = tc::fadd2(rs4[c & 3], tc::f2_pack(p0, p1));
          pk[c] = tc::pack_bf16x2(p0, p1);
        }
        tc::st32(t_s + 32 * half, pk);
      }
      const uint64_t r01 = tc::fadd2(tc::fadd2(rs4[0], rs4[1]), tc::fadd2(rs4[2], rs4[3]));
      const float rs = tc::f2_lo(r01) + tc::f2_hi(r01);
      l_run = l_run * alpha + rs;
      m_run = m_use;
      if (j > 0 && rescale) {
        // O_X may only be touched once PV_X(j-1) has finished.  It has: the
        // commit behind s_full (waited for above) tracks every MMA its thread
        // issued before S_X(j), PV_X(j-1) included.
#pragma unroll
        for (int c4 = 0; c4 < kD / 32; ++c4) {
          float o[32];
          tc::ld32(t_o + 32 * c4, reinterpret_cast<uint32_t *>(o));
          tc::wait_ld();
          const uint64_t a2 = tc::f2_pack(alpha, alpha);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint64_t r = tc::fmul2(tc::f2_pack(o[2 * c], o[2 * c + 1]), a2);
            o[2 * c] = tc::f2_lo(r);
            o[2 * c + 1] = tc::f2_hi(r);
          }
          tc::st32(t_o + 32 * c4, reinterpret_cast<const uint32_t *>(o));
        }
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[x]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && x < ntiles && wait_bar(&sm.o_final[x], 0, v.err, dead)) {
      tc::fence_after_sync();
      const int qi = qt * kTile + r;
      const float inv = 1.f / l_run;
      __nv_bfloat16 *dst = a.out + ((int64_t)(tok0 + qi) * v.H + h) * kD;
#pragma unroll
      for (int c4 = 0; c4 < kD / 32; ++c4) {
        float o[32];
        tc::ld32(t_o + 32 * c4, reinterpret_cast<uint32_t *>(o));
        tc::wait_ld();
        if (qi < P) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = tc::pack_bf16x2(o[2 * c] * inv, o[2 * c + 1] * inv);
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c4);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
    }
    // ragged last prompt tile (query tile qt of this warpgroup): rows
    // [qt * 128, P) of its K / V into the cache, from its ring slots
    const int rem = P - qt * kTile;
    if (ok && x < ntiles && rem > 0 && rem < kTile && (a.store_k || a.store_v)) {
      const int it = qt - j0;  // its load index in both rings
      const int ks = it % kKStages, vs = it % kVStages;
      const bool kr = !a.store_k || wait_bar(&sm.k_full[ks], (it / kKStages) & 1, v.err, dead);
      const bool vr = !a.store_v || wait_bar(&sm.v_full[vs], (it / kVStages) & 1, v.err, dead);
      if (kr && vr && r < rem) {
        const int64_t grow = crow0 + (int64_t)qt * kTile + r;
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const uint32_t off = (uint32_t)(c >> 3) * kHalfBytes + (uint32_t)r * 128u +
                               ((uint32_t)((c & 7) ^ (r & 7)) << 4);
          if (a.store_k)
            *reinterpret_cast<uint4 *>(a.kc + grow * kD + 8 * c) =
                *reinterpret_cast<const uint4 *>(sm.k[ks] + off);
          if (a.store_v)
            *reinterpret_cast<uint4 *>(a.vc + grow * kD + 8 * c) =
                *reinterpret_cast<const uint4 *>(sm.v[vs] + off);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kMmaWarp) tc::tmem_dealloc(tbase, kTmemCols);
}

// [tokens][H * 128] bf16 activations, 64 x 128 boxes, 128-byte swizzle.
bool make_tmap(CUtensorMap *m, const void *base, int64_t tokens, int H) {
  return make_tmap_bf16(m, base, tokens, H, kTile);
}

}  // namespace

cudaError_t launch_prefill_tc(const DeviceView &v, const void *q, const void *k, const void *vv,
                              void *out, const int4 *blocks, int n_blocks, void *kc, void *vc,
                              int k_from_cache, int64_t kc_rows, cudaStream_t s) {
  if (n_blocks == 0) return cudaSuccess;
  if (v.D != kD || v.dtype != RSWA_BF16) return cudaErrorInvalidValue;
  if (!kc || !vc || kc_rows < 1 || kc_rows >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tkc, tvc;
  // the caches as [kc_rows][1 x 128]: the same encoding with H = 1
  const bool k_ok = k_from_cache ? make_tmap(&tk, kc, kc_rows, 1)
                                 : make_tmap(&tk, k, v.total_tokens, v.H);
  if (!make_tmap(&tq, q, v.total_tokens, v.H) || !k_ok ||
      !make_tmap(&tv, vv, v.total_tokens, v.H) || !make_tmap(&tkc, kc, kc_rows, 1) ||
      !make_tmap(&tvc, vc, kc_rows, 1))
    return cudaErrorInvalidValue;
  const int smem = (int)sizeof(PrefillSmem) + 1024;
  // the attribute holds per device for the life of the process: set it once
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // the register split inside the kernel assumes kLaunchRegs per thread at
    // launch; with fewer, its setmaxnreg.inc could never be satisfied
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, prefill_tc_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  // RoPE: the rotated keys are in the cache already; only V is stored
  PrefillTcArgs args{v,  blocks, (__nv_bfloat16 *)out, (__nv_bfloat16 *)kc, (__nv_bfloat16 *)vc,
                     k_from_cache, k_from_cache ? 0 : 1, 1};
  prefill_tc_kernel<<<n_blocks, kThreads, smem, s>>>(tq, tk, tv, tkc, tvc, args);
  return cudaGetLastError();
}

}  // namespace rswa
