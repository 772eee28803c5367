// Non-causal softmax attention on the 5th-generation tensor cores (tcgen05).
//
// What it computes (API page "mstar.model.components.distributed.
// sequence_parallel", ulysses_attention / run_attention; non-causal as in
// "deepspeed/sequence/autosp_vit.py"): for every (batch, head) of the launch,
//   O = softmax(Q K^T * scale) V   over all T' tokens,
// with 16-bit inputs, fp32 scores and accumulators, P rounded to the input
// type for the P.V product, and O rounded once at the end. The epilogue writes
// each output row straight to its destination through an AttnOut table; for
// the Ulysses block that is the sequence shard of the rank owning the row's
// token (the head->seq exchange, fused).
//
// Grouped-query attention: query head h reads k/v head
// (q_head_base + h) / kv_group - kv_head_base of the k/v views.
//
// Ulysses + Ring hybrid (the RING instantiation): query rows come in groups
// and keys in blocks; a CTA's query tile lies in one group g, and it takes
// the key blocks in ring order g, g-1, ... (its own block first), each cut
// into 256-key tiles with the block's ragged last tile masked. The online
// softmax state (row maximum m, denominator l, O) carries across blocks: it is
// the ring's log-sum-exp merge, done one tile at a time. Optionally every
// row's log-sum-exp, (m + log2 l) ln 2, is written out.
//
// One CTA computes one 128-row query tile of one (batch, head), walking the
// keys in tiles of 256 (S = Q K^T is one M128 N256 MMA per 16 columns of D,
// the shape that runs the tensor core at its full rate):
//   warp 16     TMA producer: Q once; K in atom-column blocks (256 keys x one
//               swizzle atom of D) and V in half tiles (128 keys x D), each
//               into its own ring of shared-memory slots
//   warp 17     TMEM allocator and MMA issuer (one thread):
//                 S  = Q K_{j+1}^T  (SS)          -> TMEM S (issued as soon as the
//                                                    softmax has loaded S_j)
//                 O += P_j V_j      (TS: P in TMEM) -> TMEM O
//               every K block / V half is released by its own commit
//   warps 0-15  softmax: warps w, w+4, w+8, w+12 own query rows 32(w%4)..+32
//               (TMEM lane = row), each taking 64 of the 256 key columns;
//               partial row maxima are swapped through shared memory; online
//               softmax in the log2 domain; O is rescaled in TMEM only when a
//               row maximum grows by more than 2^8, otherwise the stale
//               maximum is kept (exact: the final division uses the same
//               maximum for numerator and denominator).
// TMEM columns: S [0,256), O [256,256+D), P [384,512) (256 keys, two per column).
//
// attn_tc_persistent_kernel runs the same steps with a grid of at most one
// CTA per SM, each CTA walking several (query tile, batch, head) items; the
// host takes it for short key sequences (at most 16 key tiles, where a CTA's
// fixed costs weigh most) or when the caller caps the CTA count.
#include <cmath>
#include <cstdio>

#include <cuda_fp16.h>

#include "device_common.cuh"
#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_attn_error;   // first wait that ran out (site code), 0 if none
__device__ uint32_t g_attn_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

// Pipeline trace (built only with -DUSP_TRACE): clock64() at pipeline events
// of one CTA, [event][key tile]; read with usp_debug_read_trace.
#ifdef USP_TRACE
constexpr int kTraceEvents = 14, kTraceTiles = 256;
__device__ unsigned long long g_trace[kTraceEvents][kTraceTiles];
#define USP_TRACE_EV(ev, j)                                                             \
  do {                                                                                  \
    if (trace_cta && (j) < kTraceTiles) g_trace[(ev)][(j)] = clock64();                 \
  } while (0)
#else
#define USP_TRACE_EV(ev, j) \
  do {                      \
  } while (0)
#endif

namespace {

constexpr int kBM = 128;                 // query rows per CTA
constexpr int kBN = 256;                 // keys per tile
constexpr int kParts = 4;                // softmax warps per TMEM lane quarter
constexpr int kCols = kBN / kParts;      // key columns per softmax thread
constexpr int kSoftmaxWarps = 4 * kParts;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr int kMaxVSlots = 4;            // V half-tile slots at most (the Cfg picks 2 or 4)
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s: only a broken pipeline waits this long
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s to let in-flight copies land on abort
constexpr float kRescaleThreshold = 8.0f;          // log2 units
#ifndef USP_PERSIST_MAX_TILES
#define USP_PERSIST_MAX_TILES 16
#endif
constexpr int kPersistMaxTiles = USP_PERSIST_MAX_TILES;  // key tiles per item up to which CTAs are persistent

template <int D>
struct Cfg {
  static constexpr int ATOM = (D % 64 == 0) ? 64 : ((D % 32 == 0) ? 32 : 16);  // elements per swizzle row
  static constexpr int NATOM = D / ATOM;
  static constexpr int ROWB = ATOM * 2;                // bytes per row of one atom block
  static constexpr uint32_t SBO = 8 * ROWB;            // 8-row core-matrix group stride
  static constexpr uint32_t LAYOUT = (ATOM == 64) ? 2u : ((ATOM == 32) ? 4u : 6u);
  static constexpr int Q_BYTES = kBM * D * 2;          // NATOM blocks of [128 rows][ROWB]
  static constexpr int KUNIT_BYTES = kBN * ROWB;       // one atom block of a 256-key K tile
  static constexpr int KSLOTS = NATOM + 1 < 2 ? 2 : NATOM + 1;
  static constexpr int VHALF_BYTES = (kBN / 2) * D * 2;  // NATOM blocks of [128 keys][ROWB]
  static constexpr int VBLOCK_BYTES = (kBN / 2) * ROWB;
  static constexpr int KSTEPS_PER_ATOM = ATOM / 16;
  static constexpr int BASE_BYTES = Q_BYTES + KSLOTS * KUNIT_BYTES + 1024 + 5120;
  // V half tiles in flight: two tiles ahead where shared memory allows (every
  // head_dim below 128), one tile ahead otherwise.
  static constexpr int VSLOTS = BASE_BYTES + 4 * VHALF_BYTES <= 232448 ? 4 : 2;
  static constexpr int SMEM_BYTES = BASE_BYTES + VSLOTS * VHALF_BYTES;
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[9], k_empty[9];
  uint64_t v_full[kMaxVSlots], v_empty[kMaxVSlots];
  uint64_t s_full, s_empty, p_full, pv_done;
  uint64_t o_full, o_empty, drain;
  uint64_t xbar[4];               // partial-maximum exchange among the four warps of a lane quarter
  uint32_t tmem_base;
  int abort;
  float xch[2 * kParts * kBM];    // [tile parity][part][row]
};

static_assert(sizeof(Bars) + 8 <= 5120, "barrier block outgrew its shared-memory reservation");

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v;   // boxes: Q 128 rows, K 256 rows, V 128 rows
  AttnOut out;
  float* lse;                     // optional [head][batch][tokens], natural log
  int64_t lse_ext;                // its elements (bounds-checking builds)
  int32_t tokens, batch, n_heads, kv_tokens;
  int32_t kv_group, q_head_base, kv_head_base, pad1;  // k/v head of query head h: (q_head_base + h) / kv_group - kv_head_base
  float scale_log2;
  int32_t n_qgroups, n_kvblocks;
  int32_t n_items;                // (query tile, batch, head) work items; CTA c takes c, c + gridDim.x, ...
  int32_t q_start[USP_MAX_WORLD + 1];
  int32_t q_tile_prefix[USP_MAX_WORLD + 1];
  int32_t kv_start[USP_MAX_WORLD + 1];
  uint16_t heads[USP_MAX_HEADS];
};

// Key tile j of query group g: key blocks are taken in ring order g, g-1, ...
// (mod n_kvblocks), each cut into tiles of kBN keys, the last one ragged.
// Returns the tile's first key row and the number of its keys that belong to
// its block (the rest are masked).
struct KeyTile {
  int key0;
  int valid;
};

__device__ __forceinline__ KeyTile key_tile(const TcParams& p, int g, int j) {
  const int nb = p.n_kvblocks;
  int blk = g % nb;
  for (int s = 0; s < nb; ++s) {
    const int len = p.kv_start[blk + 1] - p.kv_start[blk];
    const int nt = (len + kBN - 1) / kBN;
    if (j < nt) return KeyTile{p.kv_start[blk] + j * kBN, len - j * kBN};
    j -= nt;
    blk = blk == 0 ? nb - 1 : blk - 1;
  }
  return KeyTile{0, 0};  // not reached for j < the group's tile count
}

// One work item: a 128-row query tile of one (batch, head). Item i is query
// tile i % nq of (batch, head) pair i / nq, nq = query tiles per pair, so the
// CTAs that run at the same time share the K/V of one head through L2.
struct Item {
  int b, hm, hk;   // batch, query head, k/v head in the k/v view
  int g;           // query group (hybrid plans; 0 otherwise)
  int row0;        // first query row of the tile
};

template <bool RING>
__device__ __forceinline__ Item decode_item(const TcParams& p, int item) {
  const int nq = p.q_tile_prefix[p.n_qgroups];
  const int bh = item / nq;
  const int qtile = item - bh * nq;
  const int hi = bh / p.batch;
  Item I;
  I.b = bh - hi * p.batch;
  I.hm = p.heads[hi];
  I.hk = (p.q_head_base + I.hm) / p.kv_group - p.kv_head_base;  // grouped-query attention
  I.g = 0;
  if constexpr (RING) {
    while (I.g + 1 < p.n_qgroups && qtile >= p.q_tile_prefix[I.g + 1]) ++I.g;
    I.row0 = p.q_start[I.g] + (qtile - p.q_tile_prefix[I.g]) * kBM;
  } else {
    I.row0 = qtile * kBM;
  }
  return I;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool bf16) {
  return bf16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}
template <int D, bool BF16, bool RING>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::Q_BYTES;
  uint8_t* sV = sK + C::KSLOTS * C::KUNIT_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(sV + C::VSLOTS * C::VHALF_BYTES);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qtile = blockIdx.x;
  const int hi = blockIdx.y / p.batch;
  const int b = blockIdx.y - hi * p.batch;
  const int hm = p.heads[hi];
  const int hk = (p.q_head_base + hm) / p.kv_group - p.kv_head_base;  // grouped-query attention
  const int T = p.tokens;  // query rows; the plain kernel also takes them as keys
  auto group_of_cta = [&]() {
    int g = 0;
    if constexpr (RING)
      while (g + 1 < p.n_qgroups && static_cast<int>(blockIdx.x) >= p.q_tile_prefix[g + 1]) ++g;
    return g;
  };
  auto first_row = [&](int g) {
    if constexpr (RING) return p.q_start[g] + (static_cast<int>(blockIdx.x) - p.q_tile_prefix[g]) * kBM;
    return static_cast<int>(blockIdx.x) * kBM;
  };
  const int ntiles = [&]() {  // key tiles over all blocks
    if constexpr (RING) {
      int n = 0;
      for (int k = 0; k < p.n_kvblocks; ++k) n += (p.kv_start[k + 1] - p.kv_start[k] + kBN - 1) / kBN;
      return n;
    }
    return (T + kBN - 1) / kBN;
  }();
#ifdef USP_TRACE
  const bool trace_cta = blockIdx.x == 7 && blockIdx.y == 0;
#endif

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::KSLOTS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::VSLOTS; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_empty, kSoftmaxThreads);
    mbar_init(&bars->p_full, kSoftmaxThreads);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->xbar[q], 32 * kParts);
    // An earlier launch or CTA recorded an error: this CTA does no work.
    bars->abort = (*reinterpret_cast<volatile uint32_t*>(&g_attn_error) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const bool skip = bars->abort != 0;  // uniform: read after the barrier, before any wait

  if (skip) {
    // fall through to the common exit
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int g = 0;
      if constexpr (RING) g = group_of_cta();
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
      for (int a = 0; a < C::NATOM; ++a)
        tma_load_4d(&p.tm_q, &bars->q_full, sQ + a * kBM * C::ROWB, a * C::ATOM, hm, RING ? first_row(g) : qtile * kBM,
                    b);
      // Unit n of K is atom block n % NATOM of key tile n / NATOM; half m of V is
      // keys [128(m%2), +128) of tile m / 2. With one tile of V slots they are
      // issued in the order the tensor core consumes them (K of tile j+1
      // before V of tile j); with two, V of tile j goes first (below).
      auto load_k = [&](int n) -> bool {
        const int st = n % C::KSLOTS;
        if (n >= C::KSLOTS &&
            !mbar_wait(&bars->k_empty[st], ((n / C::KSLOTS) - 1) & 1, abort_flag, &g_attn_error, 10, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->k_full[st], C::KUNIT_BYTES);
        const int a = n % C::NATOM;
        const int key0 = RING ? key_tile(p, g, n / C::NATOM).key0 : (n / C::NATOM) * kBN;
        tma_load_4d(&p.tm_k, &bars->k_full[st], sK + st * C::KUNIT_BYTES, a * C::ATOM, hk, key0, b);
        return true;
      };
      auto load_v = [&](int m) -> bool {
        const int st = m % C::VSLOTS;
        if (m >= C::VSLOTS &&
            !mbar_wait(&bars->v_empty[st], ((m / C::VSLOTS) - 1) & 1, abort_flag, &g_attn_error, 11, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->v_full[st], C::VHALF_BYTES);
        const int key0 = (RING ? key_tile(p, g, m / 2).key0 : (m / 2) * kBN) + (m % 2) * (kBN / 2);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_v, &bars->v_full[st], sV + st * C::VHALF_BYTES + a * C::VBLOCK_BYTES, a * C::ATOM, hk,
                      key0, b);
        return true;
      };
      int nk = 0, nv = 0;  // units issued
      bool go = true;
      for (int a = 0; go && a < C::NATOM; ++a) {
        go = load_k(nk);
        nk += go;
      }
      // With two tiles of V slots, V of tile j goes first: its slot was freed
      // by P V two tiles back, while K of tile j+1 waits for Q K_j^T.
      constexpr bool kVFirst = C::VSLOTS >= 4;
      for (int j = 0; go && j < ntiles; ++j) {
        if constexpr (kVFirst) {
          for (int h = 0; go && h < 2; ++h) {
            go = load_v(nv);
            nv += go;
          }
          USP_TRACE_EV(1, j);
        }
        if (j + 1 < ntiles)
          for (int a = 0; go && a < C::NATOM; ++a) {
            go = load_k(nk);
            nk += go;
          }
        USP_TRACE_EV(0, j + 1);
        if constexpr (!kVFirst) {
          for (int h = 0; go && h < 2; ++h) {
            go = load_v(nv);
            nv += go;
          }
          USP_TRACE_EV(1, j);
        }
      }
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        for (int n = (nk > C::KSLOTS ? nk - C::KSLOTS : 0); n < nk; ++n)
          mbar_wait_drain(&bars->k_full[n % C::KSLOTS], (n / C::KSLOTS) & 1, kDrainLimitNs);
        for (int m = (nv > C::VSLOTS ? nv - C::VSLOTS : 0); m < nv; ++m)
          mbar_wait_drain(&bars->v_full[m % C::VSLOTS], (m / C::VSLOTS) & 1, kDrainLimitNs);
        mbar_wait_drain(&bars->q_full, 0, kDrainLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_f16(kBM, kBN, BF16, false);
      const uint32_t idesc_pv = make_idesc_f16(kBM, D, BF16, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, &g_attn_error, 20, kWaitLimitNs);
      tc_fence_after();
      // S = Q K_j^T, one K atom block at a time, each block released by its own commit.
      auto issue_qk = [&](int j) -> bool {
        for (int a = 0; a < C::NATOM; ++a) {
          const int n = j * C::NATOM + a;
          const int st = n % C::KSLOTS;
          if (!mbar_wait(&bars->k_full[st], (n / C::KSLOTS) & 1, abort_flag, &g_attn_error, 23, kWaitLimitNs))
            return false;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS_PER_ATOM; ++ks) {
            const uint32_t qoff = a * kBM * C::ROWB + ks * 32;
            const uint64_t adesc = make_smem_desc(q_addr + qoff, 16, C::SBO, C::LAYOUT);
            const uint64_t bdesc = make_smem_desc(k_addr + st * C::KUNIT_BYTES + ks * 32, 16, C::SBO, C::LAYOUT);
            umma_ss(tmem + kColS, adesc, bdesc, idesc_qk, (a > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->k_empty[st]);
        }
        umma_commit(&bars->s_full);
        USP_TRACE_EV(2, j);
        return true;
      };
      // O += P_j V_j, one V half (128 keys) at a time.
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(&bars->p_full, j & 1, abort_flag, &g_attn_error, 22, kWaitLimitNs)) return false;
        USP_TRACE_EV(3, j);
        for (int h = 0; h < 2; ++h) {
          const int m = 2 * j + h;
          const int st = m % C::VSLOTS;
          if (!mbar_wait(&bars->v_full[st], (m / C::VSLOTS) & 1, abort_flag, &g_attn_error, 21, kWaitLimitNs))
            return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk) {
            const uint64_t bdesc = make_smem_desc(v_addr + st * C::VHALF_BYTES + kk * 16 * C::ROWB, C::VBLOCK_BYTES,
                                                  C::SBO, C::LAYOUT);
            umma_ts(tmem + kColO, tmem + kColP + h * (kBN / 4) + kk * 8, bdesc, idesc_pv, (j > 0 || h > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->v_empty[st]);
        }
        umma_commit(&bars->pv_done);
        USP_TRACE_EV(4, j);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles) {
          // S is single-buffered: the next product waits until the softmax has read S_j.
          if (!mbar_wait(&bars->s_empty, j & 1, abort_flag, &g_attn_error, 24, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          if (!issue_qk(j + 1)) { ok = false; break; }
        }
        if (!issue_pv(j)) { ok = false; break; }
      }
      if (ok) umma_commit(&bars->o_full);
      // All MMAs this thread issued must finish before TMEM is released.
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int part = warp >> 2;                      // 0..kParts-1: key columns [kCols*part, +kCols)
    const int row = quarter * 32 + lane;             // TMEM lane = query row in the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    constexpr int kOChunks = D / 16;                 // O chunk c belongs to part c % kParts
    float* xch = bars->xch;                          // [parity][part][row]
    uint64_t* xbar = &bars->xbar[quarter];
    const float sl2 = p.scale_log2;
    int kb_blk = 0, kb_left = 0;
    if constexpr (RING) {
      kb_blk = group_of_cta() % p.n_kvblocks;
      kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
    }
    float m = -INFINITY;  // running maximum, log2 domain (identical in the four parts)
    float l = 0.f;        // this part's running denominator
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort_flag, &g_attn_error, 30, kWaitLimitNs))) { ok = false; break; }
      if (threadIdx.x == 0) USP_TRACE_EV(5, j);
      tc_fence_after();
      uint32_t sr[kCols];
      const uint32_t scol = lane_addr + kColS + part * kCols;
#pragma unroll
      for (int c = 0; c < kCols; c += 32) tmem_ld32(scol + c, sr + c);
      tmem_wait_ld();
      if (threadIdx.x == 0) USP_TRACE_EV(6, j);
      tc_fence_before();
      mbar_arrive(&bars->s_empty);

      float* s = reinterpret_cast<float*>(sr);
      int valid;  // valid columns of this part (>= kCols: all)
      if constexpr (RING) valid = kb_left - part * kCols;
      else valid = T - j * kBN - part * kCols;
      if (valid < kCols) {
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      // Partial row maximum: four independent three-input chains, then a tree.
      float mx4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a = fmaxf(s[i], s[i + 4]);
#pragma unroll
        for (int c = i + 8; c < kCols; c += 8) a = max3(a, s[c], s[c + 4]);
        mx4[i] = a;
      }
      const float pm = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      // Swap partial maxima with the other three parts of this lane quarter.
      float* xrow = xch + (j & 1) * kParts * kBM + row;
      xrow[part * kBM] = pm;
      mbar_arrive(xbar);
      if (!__all_sync(0xffffffffu, mbar_wait(xbar, j & 1, abort_flag, &g_attn_error, 34, kWaitLimitNs))) { ok = false; break; }
      const float mx = max3(fmaxf(xrow[0], xrow[kBM]), xrow[2 * kBM], xrow[3 * kBM]);
      if (threadIdx.x == 0) USP_TRACE_EV(7, j);
      const float m_new = fmaxf(m, mx * sl2);
      if (j == 0) {
        m = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
        // O holds sum_{i<j} exp2(s_i - m) v_i; bring it to the new maximum.
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (j - 1) & 1, abort_flag, &g_attn_error, 31, kWaitLimitNs))) { ok = false; break; }
        tc_fence_after();
        const float alpha = ex2_approx(m - m_new);
        m = m_new;
        l *= alpha;
        for (int c = part; c < kOChunks; c += kParts) {
          uint32_t o[16];
          tmem_ld16(lane_addr + kColO + c * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(lane_addr + kColO + c * 16, o);
        }
        tmem_wait_st();
      }
      // p = 2^(s*scale*log2e - m), packed to the input type for the P.V product.
      // Masked entries (s = -inf) give exactly 0.
      uint32_t pk[kCols / 2];
      float psum;
      {
        // One FFMA, one MUFU exp2 and one FADD per element. Full parts and
        // parts with masked columns take separate (identical) loops: the
        // split lets the compiler allocate the loop without a spill.
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float negm = -m;
        if (valid >= kCols) {
#pragma unroll
          for (int c = 0; c < kCols; c += 2) {
            const float p0 = ex2_approx(fmaf(s[c], sl2, negm));
            const float p1 = ex2_approx(fmaf(s[c + 1], sl2, negm));
            acc[c & 7] += p0;
            acc[(c + 1) & 7] += p1;
            pk[c / 2] = pack2(p0, p1, BF16);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kCols; c += 2) {
            const float p0 = ex2_approx(fmaf(s[c], sl2, negm));
            const float p1 = ex2_approx(fmaf(s[c + 1], sl2, negm));
            acc[c & 7] += p0;
            acc[(c + 1) & 7] += p1;
            pk[c / 2] = pack2(p0, p1, BF16);
          }
        }
        psum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      }
      l += psum;
      if (threadIdx.x == 0) USP_TRACE_EV(8, j);
      // P is single-buffered: it was last read by P_{j-1} V_{j-1}.
      if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (j - 1) & 1, abort_flag, &g_attn_error, 32, kWaitLimitNs))) { ok = false; break; }
      tc_fence_after();
      tmem_st32(lane_addr + kColP + part * (kCols / 2), pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
      if (threadIdx.x == 0) USP_TRACE_EV(9, j);
      if constexpr (RING) {
        kb_left -= kBN;
        if (kb_left <= 0) {
          kb_blk = kb_blk == 0 ? p.n_kvblocks - 1 : kb_blk - 1;
          kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
        }
      }
    }
    // Combine the four parts' denominators.
    if (ok) {
      float* xrow = xch + (ntiles & 1) * kParts * kBM + row;
      xrow[part * kBM] = l;
      mbar_arrive(xbar);
      ok = __all_sync(0xffffffffu, mbar_wait(xbar, ntiles & 1, abort_flag, &g_attn_error, 35, kWaitLimitNs));
      if (ok) l = (xrow[0] + xrow[kBM]) + (xrow[2 * kBM] + xrow[3 * kBM]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort_flag, &g_attn_error, 33, kWaitLimitNs))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      int t = qtile * kBM + row;
      bool row_ok = t < T;
      if constexpr (RING) {
        const int g = group_of_cta();
        t = first_row(g) + row;
        row_ok = t < p.q_start[g + 1] && t < T;
      }
      if (p.lse != nullptr && part == 0 && row_ok) {  // sum_j exp(scale s_j) = 2^m * l
        const int64_t li = (static_cast<int64_t>(hm) * p.batch + b) * T + t;
        if (in_bounds(li, 1, p.lse_ext, 22, &g_attn_bounds)) p.lse[li] = (m + log2f(l)) * 0.69314718055994531f;
      }
      const AttnOut& out = p.out;
      // Destination(s) of this row.
      int seg_lo = 0, seg_hi = 0;
      int64_t row_in_seg = 0;
      if (row_ok) {
        if (t < out.prefix) {
          seg_lo = 0;
          seg_hi = out.nseg;
          row_in_seg = t;
        } else {
          const int64_t tok = t - out.prefix;
          int sg = 0;
          while (sg + 1 < out.nseg && tok >= out.seg_start[sg + 1]) ++sg;
          seg_lo = sg;
          seg_hi = sg + 1;
          row_in_seg = out.prefix + tok - out.seg_start[sg];
        }
      }
      for (int c = part; c < kOChunks; c += kParts) {
        uint32_t o[16];
        tmem_ld16(lane_addr + kColO + c * 16, o);
        tmem_wait_ld();
        uint4 w0, w1;
        w0.x = pack2(__uint_as_float(o[0]) * inv_l, __uint_as_float(o[1]) * inv_l, BF16);
        w0.y = pack2(__uint_as_float(o[2]) * inv_l, __uint_as_float(o[3]) * inv_l, BF16);
        w0.z = pack2(__uint_as_float(o[4]) * inv_l, __uint_as_float(o[5]) * inv_l, BF16);
        w0.w = pack2(__uint_as_float(o[6]) * inv_l, __uint_as_float(o[7]) * inv_l, BF16);
        w1.x = pack2(__uint_as_float(o[8]) * inv_l, __uint_as_float(o[9]) * inv_l, BF16);
        w1.y = pack2(__uint_as_float(o[10]) * inv_l, __uint_as_float(o[11]) * inv_l, BF16);
        w1.z = pack2(__uint_as_float(o[12]) * inv_l, __uint_as_float(o[13]) * inv_l, BF16);
        w1.w = pack2(__uint_as_float(o[14]) * inv_l, __uint_as_float(o[15]) * inv_l, BF16);
        for (int sg = seg_lo; sg < seg_hi; ++sg) {
          const int64_t rows_s = out.prefix + out.seg_len[sg];
          const int64_t elem =
              ((static_cast<int64_t>(b) * rows_s + row_in_seg) * out.out_heads + hm - out.head_base) * D + c * 16;
          if (!in_bounds(elem, 16, static_cast<int64_t>(p.batch) * rows_s * out.out_heads * D, 21, &g_attn_bounds))
            continue;
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out.seg_ptr[sg]) + elem);
          dst[0] = w0;
          dst[1] = w1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// The persistent form of the kernel above: a grid of at most one CTA per SM,
// CTA c taking items c, c + gridDim.x, ... (an item is one 128-row query tile
// of one (batch, head)). Each role runs the same per-tile steps over the
// CTA's items in order, with K/V slots, barrier phases and the exchange phase
// counted across items. Two barriers carry the hand-off between items: the
// next item's Q is loaded once q_empty says the last Q K^T of the previous
// item has completed, and the next item's first P V (which overwrites O) is
// issued once o_empty says the softmax warps have read the previous O. So an
// item's Q/K loads and first Q K^T run under the previous item's last tiles.
// It is a separate kernel because the item bookkeeping, at the 96-register
// cap of a 576-thread CTA, costs the one-item kernel a spilled register and
// about 2% on long sequences.
template <int D, bool BF16, bool RING>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_persistent_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::Q_BYTES;
  uint8_t* sV = sK + C::KSLOTS * C::KUNIT_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(sV + C::VSLOTS * C::VHALF_BYTES);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = p.tokens;  // query rows; the plain kernel also takes them as keys
  const int first_item = blockIdx.x;
  const int item_stride = gridDim.x;
  // Does this CTA have an item number `it`?
  auto has_item = [&](int it) { return first_item + it * item_stride < p.n_items; };
  const int ntiles = [&]() {  // key tiles of every item, over all blocks
    if constexpr (RING) {
      int n = 0;
      for (int k = 0; k < p.n_kvblocks; ++k) n += (p.kv_start[k + 1] - p.kv_start[k] + kBN - 1) / kBN;
      return n;
    }
    return (T + kBN - 1) / kBN;
  }();
#ifdef USP_TRACE
  const bool trace_cta = blockIdx.x == 7;
#endif

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::KSLOTS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::VSLOTS; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_empty, kSoftmaxThreads);
    mbar_init(&bars->p_full, kSoftmaxThreads);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_empty, kSoftmaxThreads);
    mbar_init(&bars->drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->xbar[q], 32 * kParts);
    // An earlier launch or CTA recorded an error: this CTA does no work.
    bars->abort = (*reinterpret_cast<volatile uint32_t*>(&g_attn_error) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const bool skip = bars->abort != 0;  // uniform: read after the barrier, before any wait

  if (skip) {
    // fall through to the common exit
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      // Q of item number `it` of this CTA; the slot is free once the previous
      // item's last Q.K^T product has completed.
      auto load_q = [&](const Item& I, int it) -> bool {
        if (it >= 1 && !mbar_wait(&bars->q_empty, (it - 1) & 1, abort_flag, &g_attn_error, 12, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_q, &bars->q_full, sQ + a * kBM * C::ROWB, a * C::ATOM, I.hm, I.row0, I.b);
        return true;
      };
      // K goes in atom-column blocks, unit n (counted over the CTA's items) into
      // slot n % KSLOTS; V in half tiles of 128 keys, half m into slot
      // m % VSLOTS. K of tile j+1 (or of the next item's first tile) and V of
      // tile j are ordered as in the one-item kernel.
      auto load_k = [&](const Item& I, int n, int j, int a) -> bool {
        const int st = n % C::KSLOTS;
        if (n >= C::KSLOTS &&
            !mbar_wait(&bars->k_empty[st], ((n / C::KSLOTS) - 1) & 1, abort_flag, &g_attn_error, 10, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->k_full[st], C::KUNIT_BYTES);
        const int key0 = RING ? key_tile(p, I.g, j).key0 : j * kBN;
        tma_load_4d(&p.tm_k, &bars->k_full[st], sK + st * C::KUNIT_BYTES, a * C::ATOM, I.hk, key0, I.b);
        return true;
      };
      auto load_v = [&](const Item& I, int m, int j, int h) -> bool {
        const int st = m % C::VSLOTS;
        if (m >= C::VSLOTS &&
            !mbar_wait(&bars->v_empty[st], ((m / C::VSLOTS) - 1) & 1, abort_flag, &g_attn_error, 11, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->v_full[st], C::VHALF_BYTES);
        const int key0 = (RING ? key_tile(p, I.g, j).key0 : j * kBN) + h * (kBN / 2);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_v, &bars->v_full[st], sV + st * C::VHALF_BYTES + a * C::VBLOCK_BYTES, a * C::ATOM, I.hk,
                      key0, I.b);
        return true;
      };
      // With two tiles of V slots, V of tile j goes first: its slot was freed
      // by P V two tiles back, while K of tile j+1 waits for Q K_j^T.
      constexpr bool kVFirst = C::VSLOTS >= 4;
      int nk = 0, nv = 0, nql = 0;  // K units, V halves and Q tiles issued
      int jg = 0;                   // key tiles over the CTA's items (trace index)
      int item = first_item;
      Item I = decode_item<RING>(p, item);
      bool go = load_q(I, 0);
      nql += go;
      for (int a = 0; go && a < C::NATOM; ++a) {
        go = load_k(I, nk, 0, a);
        nk += go;
      }
      for (int it = 0; go && has_item(it); ++it, item += item_stride) {
        const bool has_next = has_item(it + 1);
        const Item N = has_next ? decode_item<RING>(p, item + item_stride) : I;
        for (int j = 0; go && j < ntiles; ++j) {
          if constexpr (kVFirst) {
            for (int h = 0; go && h < 2; ++h) {
              go = load_v(I, nv, j, h);
              nv += go;
            }
            USP_TRACE_EV(1, jg);
          }
          if (j + 1 < ntiles) {
            for (int a = 0; go && a < C::NATOM; ++a) {
              go = load_k(I, nk, j + 1, a);
              nk += go;
            }
          } else if (has_next) {
            go = load_q(N, it + 1);
            nql += go;
            for (int a = 0; go && a < C::NATOM; ++a) {
              go = load_k(N, nk, 0, a);
              nk += go;
            }
          }
          USP_TRACE_EV(0, jg + 1);
          if constexpr (!kVFirst) {
            for (int h = 0; go && h < 2; ++h) {
              go = load_v(I, nv, j, h);
              nv += go;
            }
            USP_TRACE_EV(1, jg);
          }
          ++jg;
        }
        I = N;
      }
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        for (int n = (nk > C::KSLOTS ? nk - C::KSLOTS : 0); n < nk; ++n)
          mbar_wait_drain(&bars->k_full[n % C::KSLOTS], (n / C::KSLOTS) & 1, kDrainLimitNs);
        for (int m = (nv > C::VSLOTS ? nv - C::VSLOTS : 0); m < nv; ++m)
          mbar_wait_drain(&bars->v_full[m % C::VSLOTS], (m / C::VSLOTS) & 1, kDrainLimitNs);
        if (nql > 0) mbar_wait_drain(&bars->q_full, (nql - 1) & 1, kDrainLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_f16(kBM, kBN, BF16, false);
      const uint32_t idesc_pv = make_idesc_f16(kBM, D, BF16, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      int kc = 0, vc = 0;  // K units and V halves consumed, over the CTA's items
      // S = Q K^T for the next key tile in order, one K atom block at a time,
      // each block released by its own commit. The last tile of an item also
      // releases the Q slot.
      auto issue_qk = [&](int jg, bool last_of_item) -> bool {
        for (int a = 0; a < C::NATOM; ++a, ++kc) {
          const int st = kc % C::KSLOTS;
          if (!mbar_wait(&bars->k_full[st], (kc / C::KSLOTS) & 1, abort_flag, &g_attn_error, 23, kWaitLimitNs))
            return false;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS_PER_ATOM; ++ks) {
            const uint32_t qoff = a * kBM * C::ROWB + ks * 32;
            const uint64_t adesc = make_smem_desc(q_addr + qoff, 16, C::SBO, C::LAYOUT);
            const uint64_t bdesc = make_smem_desc(k_addr + st * C::KUNIT_BYTES + ks * 32, 16, C::SBO, C::LAYOUT);
            umma_ss(tmem + kColS, adesc, bdesc, idesc_qk, (a > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->k_empty[st]);
        }
        umma_commit(&bars->s_full);
        if (last_of_item) umma_commit(&bars->q_empty);
        USP_TRACE_EV(2, jg);
        return true;
      };
      // O += P V for key tile jg, one V half (128 keys) at a time; the first
      // tile of an item overwrites O.
      auto issue_pv = [&](int jg, bool first_of_item) -> bool {
        if (!mbar_wait(&bars->p_full, jg & 1, abort_flag, &g_attn_error, 22, kWaitLimitNs)) return false;
        USP_TRACE_EV(3, jg);
        for (int h = 0; h < 2; ++h, ++vc) {
          const int st = vc % C::VSLOTS;
          if (!mbar_wait(&bars->v_full[st], (vc / C::VSLOTS) & 1, abort_flag, &g_attn_error, 21, kWaitLimitNs))
            return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk) {
            const uint64_t bdesc = make_smem_desc(v_addr + st * C::VHALF_BYTES + kk * 16 * C::ROWB, C::VBLOCK_BYTES,
                                                  C::SBO, C::LAYOUT);
            umma_ts(tmem + kColO, tmem + kColP + h * (kBN / 4) + kk * 8, bdesc, idesc_pv,
                    (!first_of_item || h > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->v_empty[st]);
        }
        umma_commit(&bars->pv_done);
        USP_TRACE_EV(4, jg);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, &g_attn_error, 20, kWaitLimitNs);
      tc_fence_after();
      if (ok) ok = issue_qk(0, ntiles == 1);
      int jg = 0;  // key tiles over the CTA's items
      for (int it = 0; ok && has_item(it); ++it) {
        const bool has_next = has_item(it + 1);
        for (int j = 0; ok && j < ntiles; ++j, ++jg) {
          if (j + 1 < ntiles || has_next) {
            // S is single-buffered: the next product waits until the softmax has read S_j.
            if (!mbar_wait(&bars->s_empty, jg & 1, abort_flag, &g_attn_error, 24, kWaitLimitNs)) { ok = false; break; }
            tc_fence_after();
            if (j + 1 == ntiles) {  // first tile of the next item: its Q must have landed
              if (!mbar_wait(&bars->q_full, (it + 1) & 1, abort_flag, &g_attn_error, 25, kWaitLimitNs)) { ok = false; break; }
              tc_fence_after();
              ok = issue_qk(jg + 1, ntiles == 1);
            } else {
              ok = issue_qk(jg + 1, j + 2 == ntiles);
            }
            if (!ok) break;
          }
          if (j == 0 && it > 0) {
            // O is single-buffered: the softmax warps must have read the previous item's O.
            if (!mbar_wait(&bars->o_empty, (it - 1) & 1, abort_flag, &g_attn_error, 26, kWaitLimitNs)) { ok = false; break; }
            tc_fence_after();
          }
          if (!issue_pv(jg, j == 0)) { ok = false; break; }
        }
        if (ok) umma_commit(&bars->o_full);
      }
      // All MMAs this thread issued must finish before TMEM is released.
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int part = warp >> 2;                      // 0..kParts-1: key columns [kCols*part, +kCols)
    const int row = quarter * 32 + lane;             // TMEM lane = query row in the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    constexpr int kOChunks = D / 16;                 // O chunk c belongs to part c % kParts
    float* xch = bars->xch;                          // [parity][part][row]
    uint64_t* xbar = &bars->xbar[quarter];
    const float sl2 = p.scale_log2;
    bool ok = true;
    // Epilogue of item e_it (running maximum e_m, combined denominator e_l):
    // O is read from TMEM, normalised and stored to its rows' sequence shards,
    // and o_empty lets the next item's first P V overwrite O.
    auto epilogue = [&](int e_it, float e_m, float e_l) {
      tc_fence_after();
      const Item I = decode_item<RING>(p, first_item + e_it * item_stride);
      const float inv_l = 1.f / e_l;
      const int t = I.row0 + row;
      bool row_ok = t < T;
      if constexpr (RING) row_ok = t < p.q_start[I.g + 1] && t < T;
      const int b = I.b, hm = I.hm;
      if (p.lse != nullptr && part == 0 && row_ok) {  // sum_j exp(scale s_j) = 2^m * l
        const int64_t li = (static_cast<int64_t>(hm) * p.batch + b) * T + t;
        if (in_bounds(li, 1, p.lse_ext, 22, &g_attn_bounds)) p.lse[li] = (e_m + log2f(e_l)) * 0.69314718055994531f;
      }
      const AttnOut& out = p.out;
      // Destination(s) of this row.
      int seg_lo = 0, seg_hi = 0;
      int64_t row_in_seg = 0;
      if (row_ok) {
        if (t < out.prefix) {
          seg_lo = 0;
          seg_hi = out.nseg;
          row_in_seg = t;
        } else {
          const int64_t tok = t - out.prefix;
          int sg = 0;
          while (sg + 1 < out.nseg && tok >= out.seg_start[sg + 1]) ++sg;
          seg_lo = sg;
          seg_hi = sg + 1;
          row_in_seg = out.prefix + tok - out.seg_start[sg];
        }
      }
      // A warp holds 32 rows x 16 columns of each O chunk (32 bytes a row).
      // Lanes are paired per row for the stores: in round h, lane t writes
      // half t & 1 of row 16h + t/2 of the warp, so each store instruction
      // fills 16 whole 32-byte sectors instead of touching 32 half sectors.
      // Every softmax thread arrives on o_empty once it has read its last
      // chunk of O, or at once if its part holds none (head_dim < 64).
      if (part >= kOChunks) {
        tc_fence_before();
        mbar_arrive(&bars->o_empty);
      }
      for (int c = part; c < kOChunks; c += kParts) {
        uint32_t o[16];
        tmem_ld16(lane_addr + kColO + c * 16, o);
        tmem_wait_ld();
        if (c + kParts >= kOChunks) {  // this thread's last chunk: O is free for the next item
          tc_fence_before();
          mbar_arrive(&bars->o_empty);
        }
        uint4 w0, w1;
        w0.x = pack2(__uint_as_float(o[0]) * inv_l, __uint_as_float(o[1]) * inv_l, BF16);
        w0.y = pack2(__uint_as_float(o[2]) * inv_l, __uint_as_float(o[3]) * inv_l, BF16);
        w0.z = pack2(__uint_as_float(o[4]) * inv_l, __uint_as_float(o[5]) * inv_l, BF16);
        w0.w = pack2(__uint_as_float(o[6]) * inv_l, __uint_as_float(o[7]) * inv_l, BF16);
        w1.x = pack2(__uint_as_float(o[8]) * inv_l, __uint_as_float(o[9]) * inv_l, BF16);
        w1.y = pack2(__uint_as_float(o[10]) * inv_l, __uint_as_float(o[11]) * inv_l, BF16);
        w1.z = pack2(__uint_as_float(o[12]) * inv_l, __uint_as_float(o[13]) * inv_l, BF16);
        w1.w = pack2(__uint_as_float(o[14]) * inv_l, __uint_as_float(o[15]) * inv_l, BF16);
        const bool hi_half = lane & 1;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // Row src's two halves come from lane src (which holds that row);
          // this lane keeps the half it writes.
          const int src = 16 * h + (lane >> 1);
          uint4 a, v;
          a.x = __shfl_sync(0xffffffffu, w0.x, src);
          a.y = __shfl_sync(0xffffffffu, w0.y, src);
          a.z = __shfl_sync(0xffffffffu, w0.z, src);
          a.w = __shfl_sync(0xffffffffu, w0.w, src);
          v.x = __shfl_sync(0xffffffffu, w1.x, src);
          v.y = __shfl_sync(0xffffffffu, w1.y, src);
          v.z = __shfl_sync(0xffffffffu, w1.z, src);
          v.w = __shfl_sync(0xffffffffu, w1.w, src);
          const uint4 val = hi_half ? v : a;
          const int lo = __shfl_sync(0xffffffffu, seg_lo, src);
          const int hi = __shfl_sync(0xffffffffu, seg_hi, src);
          const int64_t r_in = __shfl_sync(0xffffffffu, row_in_seg, src);
          for (int sg = lo; sg < hi; ++sg) {
            const int64_t rows_s = out.prefix + out.seg_len[sg];
            const int64_t elem =
                ((static_cast<int64_t>(b) * rows_s + r_in) * out.out_heads + hm - out.head_base) * D + c * 16 +
                (lane & 1) * 8;
            if (!in_bounds(elem, 8, static_cast<int64_t>(p.batch) * rows_s * out.out_heads * D, 21, &g_attn_bounds))
              continue;
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out.seg_ptr[sg]) + elem) = val;
          }
        }
      }
      if (threadIdx.x == 0) USP_TRACE_EV(12, e_it);
    };
    // An item's epilogue is deferred to the first tile of the next item: that
    // tile's softmax runs while the item's last P V completes, and its P is
    // stored (so the next P V, which overwrites O, can start) right after.
    float m_prev = 0.f, l_prev = 1.f;
    int last_it = -1;
    // jg = jg0 + j counts key tiles over the CTA's items: the phase of s_full,
    // p_full and pv_done. The quarter's exchange barrier completes once per
    // tile and once per item (the denominator combine), so its phase is jg + it.
    int jg0 = 0;
    for (int it = 0; ok && has_item(it); ++it, jg0 += ntiles) {
      int kb_blk = 0, kb_left = 0;
      if constexpr (RING) {
        kb_blk = decode_item<RING>(p, first_item + it * item_stride).g % p.n_kvblocks;
        kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
      }
      float m = -INFINITY;  // running maximum, log2 domain (identical in the four parts)
      float l = 0.f;        // this part's running denominator
      for (int j = 0; j < ntiles; ++j) {
        const int jg = jg0 + j;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, jg & 1, abort_flag, &g_attn_error, 30, kWaitLimitNs))) { ok = false; break; }
        if (threadIdx.x == 0) USP_TRACE_EV(5, jg);
        tc_fence_after();
        uint32_t sr[kCols];
        const uint32_t scol = lane_addr + kColS + part * kCols;
  #pragma unroll
        for (int c = 0; c < kCols; c += 32) tmem_ld32(scol + c, sr + c);
        tmem_wait_ld();
        if (threadIdx.x == 0) USP_TRACE_EV(6, jg);
        tc_fence_before();
        mbar_arrive(&bars->s_empty);

        float* s = reinterpret_cast<float*>(sr);
        int valid;  // valid columns of this part (>= kCols: all)
        if constexpr (RING) valid = kb_left - part * kCols;
        else valid = T - j * kBN - part * kCols;
        if (valid < kCols) {
  #pragma unroll
          for (int c = 0; c < kCols; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        // Partial row maximum: four independent three-input chains, then a tree.
        float mx4[4];
  #pragma unroll
        for (int i = 0; i < 4; ++i) {
          float a = fmaxf(s[i], s[i + 4]);
  #pragma unroll
          for (int c = i + 8; c < kCols; c += 8) a = max3(a, s[c], s[c + 4]);
          mx4[i] = a;
        }
        const float pm = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
        // Swap partial maxima with the other three parts of this lane quarter.
        const int xp = jg + it;
        float* xrow = xch + (xp & 1) * kParts * kBM + row;
        xrow[part * kBM] = pm;
        mbar_arrive(xbar);
        if (!__all_sync(0xffffffffu, mbar_wait(xbar, xp & 1, abort_flag, &g_attn_error, 34, kWaitLimitNs))) { ok = false; break; }
        const float mx = max3(fmaxf(xrow[0], xrow[kBM]), xrow[2 * kBM], xrow[3 * kBM]);
        if (threadIdx.x == 0) USP_TRACE_EV(7, jg);
        const float m_new = fmaxf(m, mx * sl2);
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
          // O holds sum_{i<j} exp2(s_i - m) v_i; bring it to the new maximum.
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (jg - 1) & 1, abort_flag, &g_attn_error, 31, kWaitLimitNs))) { ok = false; break; }
          tc_fence_after();
          const float alpha = ex2_approx(m - m_new);
          m = m_new;
          l *= alpha;
          for (int c = part; c < kOChunks; c += kParts) {
            uint32_t o[16];
            tmem_ld16(lane_addr + kColO + c * 16, o);
            tmem_wait_ld();
  #pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(lane_addr + kColO + c * 16, o);
          }
          tmem_wait_st();
        }
        // p = 2^(s*scale*log2e - m), packed to the input type for the P.V product.
        // Masked entries (s = -inf) give exactly 0.
        uint32_t pk[kCols / 2];
        float psum;
        {
          // One FFMA, one MUFU exp2 and one FADD per element. Full parts and
          // parts with masked columns take separate (identical) loops: the
          // split lets the compiler allocate the loop without a spill.
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          const float negm = -m;
          if (valid >= kCols) {
  #pragma unroll
            for (int c = 0; c < kCols; c += 2) {
              const float p0 = ex2_approx(fmaf(s[c], sl2, negm));
              const float p1 = ex2_approx(fmaf(s[c + 1], sl2, negm));
              acc[c & 7] += p0;
              acc[(c + 1) & 7] += p1;
              pk[c / 2] = pack2(p0, p1, BF16);
            }
          } else {
  #pragma unroll
            for (int c = 0; c < kCols; c += 2) {
              const float p0 = ex2_approx(fmaf(s[c], sl2, negm));
              const float p1 = ex2_approx(fmaf(s[c + 1], sl2, negm));
              acc[c & 7] += p0;
              acc[(c + 1) & 7] += p1;
              pk[c / 2] = pack2(p0, p1, BF16);
            }
          }
          psum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        }
        l += psum;
        if (threadIdx.x == 0) USP_TRACE_EV(8, jg);
        // P is single-buffered: it was last read by the previous tile's P V.
        if (jg >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (jg - 1) & 1, abort_flag, &g_attn_error, 32, kWaitLimitNs))) { ok = false; break; }
        if (j == 0 && it > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full, (it - 1) & 1, abort_flag, &g_attn_error, 33, kWaitLimitNs))) { ok = false; break; }
          if (threadIdx.x == 0) USP_TRACE_EV(11, it - 1);
          epilogue(it - 1, m_prev, l_prev);
        }
        tc_fence_after();
        tmem_st32(lane_addr + kColP + part * (kCols / 2), pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full);
        if (threadIdx.x == 0) USP_TRACE_EV(9, jg);
        if constexpr (RING) {
          kb_left -= kBN;
          if (kb_left <= 0) {
            kb_blk = kb_blk == 0 ? p.n_kvblocks - 1 : kb_blk - 1;
            kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
          }
        }
      }
      // Combine the four parts' denominators.
      if (ok) {
        const int xp = jg0 + ntiles + it;
        float* xrow = xch + (xp & 1) * kParts * kBM + row;
        xrow[part * kBM] = l;
        mbar_arrive(xbar);
        ok = __all_sync(0xffffffffu, mbar_wait(xbar, xp & 1, abort_flag, &g_attn_error, 35, kWaitLimitNs));
        if (threadIdx.x == 0) USP_TRACE_EV(10, it);
        if (ok) l = (xrow[0] + xrow[kBM]) + (xrow[2 * kBM] + xrow[3 * kBM]);
      }
      m_prev = m;
      l_prev = l;
      last_it = it;
    }
    // The last item's epilogue.
    if (ok && last_it >= 0 &&
        __all_sync(0xffffffffu, mbar_wait(&bars->o_full, last_it & 1, abort_flag, &g_attn_error, 33, kWaitLimitNs))) {
      if (threadIdx.x == 0) USP_TRACE_EV(11, last_it);
      epilogue(last_it, m_prev, l_prev);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// -------------------------------------------------------------- host side
template <int D, bool BF16>
int launch_d(const AttnLaunch& L, cudaStream_t stream) {
  using C = Cfg<D>;
  static_assert(C::SMEM_BYTES <= 232448, "shared memory above the 227 KB per-CTA limit");
  for (auto* fn : {attn_tc_kernel<D, BF16, false>, attn_tc_kernel<D, BF16, true>,
                   attn_tc_persistent_kernel<D, BF16, false>, attn_tc_persistent_kernel<D, BF16, true>})
    if (int rc = ensure_smem_limit(reinterpret_cast<const void*>(fn), C::SMEM_BYTES,
                                   "cudaFuncSetAttribute(attention smem)"))
      return rc;
  TcParams p;
  memset(&p, 0, sizeof(p));
  int rc;
  const int kv_tokens = L.kv_tokens > 0 ? L.kv_tokens : L.tokens;
  const bool ring = L.blocks.n_qgroups > 0 || L.blocks.n_kvblocks > 0;
  if (!ring && kv_tokens != L.tokens)
    return set_error(USP_ERR_INVALID_ARG, "internal: the plain attention kernel takes as many keys as queries");
  if ((rc = make_map(&p.tm_q, L.in.q, L.in.qv, L, L.tokens, C::ATOM, kBM)) != USP_OK) return rc;
  if ((rc = make_map(&p.tm_k, L.in.k, L.in.kvv, L, kv_tokens, C::ATOM, kBN)) != USP_OK) return rc;
  if ((rc = make_map(&p.tm_v, L.in.v, L.in.kvv, L, kv_tokens, C::ATOM, kBN / 2)) != USP_OK) return rc;
  if (!fill_blocks(L, kv_tokens, kBM, p.n_qgroups, p.n_kvblocks, p.q_start, p.q_tile_prefix, p.kv_start))
    return set_error(USP_ERR_INVALID_ARG, "internal: bad query-group or key-block table");
  p.kv_tokens = kv_tokens;
  p.lse = L.lse;
  p.lse_ext = static_cast<int64_t>(L.in.qv.head_extent) * L.batch * L.tokens;
  p.kv_group = L.in.kv_group;
  p.q_head_base = L.in.q_head_base;
  p.kv_head_base = L.in.kv_head_base;
  p.out = L.out;
  p.tokens = L.tokens;
  p.batch = L.batch;
  p.n_heads = L.n_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(L.scale) * 1.4426950408889634);
  for (int i = 0; i < L.n_heads; ++i) p.heads[i] = L.heads[i];
  const int64_t items = static_cast<int64_t>(p.q_tile_prefix[p.n_qgroups]) * L.batch * L.n_heads;
  if (items > INT32_MAX) return set_error(USP_ERR_UNSUPPORTED, "tcgen05 attention: %lld query tiles in one launch", (long long)items);
  p.n_items = static_cast<int32_t>(items);
  // Few key tiles per item make a CTA's fixed costs (launch, first loads, the
  // last P V and the epilogue) a large share of its time: then one CTA per SM
  // walks the items and starts each item's loads and first Q K^T under the
  // previous item's last tiles. Long key sequences keep one CTA per item, so
  // that kernels on other streams (the next head chunk's exchange) can take
  // SMs as CTAs retire. A caller's cap overrides both.
  int64_t key_tiles = 0;
  for (int k = 0; k < p.n_kvblocks; ++k) key_tiles += (p.kv_start[k + 1] - p.kv_start[k] + kBN - 1) / kBN;
  const int64_t cap = L.max_ctas > 0 ? L.max_ctas : (key_tiles <= kPersistMaxTiles ? sm_count() : items);
  if (items > cap) {
    const dim3 grid(static_cast<unsigned>(cap));
    if (ring)
      attn_tc_persistent_kernel<D, BF16, true><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
    else
      attn_tc_persistent_kernel<D, BF16, false><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  } else {
    const dim3 grid(p.q_tile_prefix[p.n_qgroups], L.batch * L.n_heads);  // one CTA per item
    if (ring)
      attn_tc_kernel<D, BF16, true><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
    else
      attn_tc_kernel<D, BF16, false><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  }
  count_launch();
  return cuda_check(cudaGetLastError(), "attention (tcgen05) launch");
}

template <bool BF16>
int launch_dtype(const AttnLaunch& L, cudaStream_t stream) {
  switch (L.head_dim) {
    case 16: return launch_d<16, BF16>(L, stream);
    case 32: return launch_d<32, BF16>(L, stream);
    case 48: return launch_d<48, BF16>(L, stream);
    case 64: return launch_d<64, BF16>(L, stream);
    case 80: return launch_d<80, BF16>(L, stream);
    case 96: return launch_d<96, BF16>(L, stream);
    case 112: return launch_d<112, BF16>(L, stream);
    case 128: return launch_d<128, BF16>(L, stream);
    default: return set_error(USP_ERR_UNSUPPORTED, "tcgen05 attention: head_dim %d not built", L.head_dim);
  }
}

__global__ void wait_timeout_probe_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up after limit_ns.
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, &g_attn_error, 99, limit_ns);
  __syncthreads();
}

}  // namespace

bool attention_tc_supported(int dtype, int head_dim) {
  return (dtype == USP_BF16 || dtype == USP_FP16) && head_dim % 16 == 0 && head_dim >= 16 && head_dim <= 128;
}

int launch_attention_tc(const AttnLaunch& L, cudaStream_t stream) {
  if (L.n_heads == 0 || L.batch == 0 || L.tokens == 0) return USP_OK;
  if (L.kernel == USP_ATTN_TWO_TILE || L.kernel == USP_ATTN_TWO_CTA) return launch_attention_pp(L, stream);
  // Automatic: long key sequences, where one CTA per query tile would be
  // launched, take the two-query-tile kernel. Short ones take the same kernel
  // with one query tile per CTA and two CTAs per SM where it is built
  // (head_dim 64 and 80), else persistent CTAs here; capped launches stay here.
  if (L.kernel == USP_ATTN_AUTO && L.max_ctas == 0 && attention_pp_supported(L.dtype, L.head_dim)) {
    const int kv_tokens = L.kv_tokens > 0 ? L.kv_tokens : L.tokens;
    int32_t nq = 0, nk = 0, q_start[USP_MAX_WORLD + 1], q_prefix[USP_MAX_WORLD + 1], kv_start[USP_MAX_WORLD + 1];
    if (fill_blocks(L, kv_tokens, kBM, nq, nk, q_start, q_prefix, kv_start)) {
      int64_t key_tiles = 0;
      for (int k = 0; k < nk; ++k) key_tiles += (kv_start[k + 1] - kv_start[k] + kBN - 1) / kBN;
      if (key_tiles > kPersistMaxTiles) return launch_attention_pp(L, stream);
      if (attention_pp_supported(L.dtype, L.head_dim, USP_ATTN_TWO_CTA)) {
        AttnLaunch two_cta = L;
        two_cta.kernel = USP_ATTN_TWO_CTA;
        return launch_attention_pp(two_cta, stream);
      }
    }
  }
  return L.dtype == USP_BF16 ? launch_dtype<true>(L, stream) : launch_dtype<false>(L, stream);
}

int read_attention_bounds(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_attn_bounds, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read attention bounds word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_attn_bounds, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset attention bounds word");
  }
  return USP_OK;
}

int read_attention_error(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_attn_error, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read device error word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_attn_error, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset device error word");
  }
  return USP_OK;
}

#ifdef USP_TRACE
extern "C" int usp_debug_read_trace(unsigned long long* out, int n) {
  const int total = kTraceEvents * kTraceTiles;
  if (n > total) n = total;
  return cudaMemcpyFromSymbol(out, g_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 5;
}
#endif

int launch_wait_timeout_probe(uint32_t limit_us, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000ull);
  count_launch();
  return cuda_check(cudaGetLastError(), "wait-timeout probe launch");
}

}  // namespace usp
