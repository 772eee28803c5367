// Non-causal softmax attention on the tcgen05 tensor cores with 128-key
// tiles: two query tiles per CTA ("ping-pong", QT = 2), or one query tile per
// CTA with two CTAs per SM (QT = 1).
//
// What it computes is exactly what attn_tc.cu computes (API page
// "mstar.model.components.distributed.sequence_parallel", ulysses_attention /
// run_attention; non-causal as in "deepspeed/sequence/autosp_vit.py"):
//   O = softmax(Q K^T * scale) V   for every (batch, head) of the launch,
// 16-bit inputs, fp32 scores and accumulators, P rounded to the input type
// for the P.V product, O rounded once at the end, each output row written
// straight to its destination through the AttnOut table (the head->seq
// exchange, fused), with the Ulysses + Ring key-block walk (RING) and
// grouped-query attention as in attn_tc.cu.
//
// How it is organised differs. A work item is QT 128-row query tiles of one
// (batch, head); a CTA walks the keys of its item in tiles of 128:
//   warps 0..4QT-1  softmax, four warps per tile: one thread per query row
//                   (TMEM lane = row), holding the row's 128 scores, so no
//                   partial maxima are exchanged between threads
//   warp 4QT        TMA producer: the item's Q tiles, then K and V tiles into rings
//   warp 4QT+1      TMEM allocator and MMA issuer (one thread), in the order
//                     S_A(0) S_B(0) | PV_A(j-1) S_A(j) PV_B(j-1) S_B(j) | ...
//                   (tile B only when QT = 2), so that while the softmax of one
//                   tile runs, the tensor core works on the other tile's products
//                   (with QT = 1, on the other CTA's).
// TMEM columns: S of tile t at 128t, O of tile t at 128 QT + 128t (D wide).
// P (128 keys, two 16-bit values per column) is written over the first 64
// columns of its tile's S, which the softmax has already read into registers,
// in two halves; the P.V products over the first half's 64 keys are issued as
// soon as that half is stored. The next S of that tile is issued only after
// the P.V that reads P, and the tensor core runs one thread's MMAs in order.
// O is rescaled in TMEM only when a row maximum grows by more than 2^8 (the
// stale maximum is kept otherwise: exact, since numerator and denominator use
// the same maximum). A tile's O is only ever written by its own P.V, which
// has completed whenever the tile's next S has (one commit covers both).
// QT = 2 launches one CTA per item. QT = 1 launches two CTAs per SM that walk
// the items; every ring stage and barrier phase follows the CTA's running tile
// count, an item's Q loads once the previous item's last S is done (q_empty),
// and its first P.V waits for the previous epilogue's reads of O (o_free).
#include <algorithm>
#include <cmath>

#include "device_common.cuh"
#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_pp_error;   // first wait that ran out (site code), 0 if none
__device__ uint32_t g_pp_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

// Pipeline trace (built only with -DUSP_TRACE): clock64() at pipeline events
// of one CTA (CTA min(7, half the grid); the grid is one-dimensional, so the
// second condition always holds), [event][the CTA's key tile, or item for the
// per-item stamps]; read with usp_debug_read_trace_pp.
#ifdef USP_TRACE
constexpr int kPpTraceEvents = 16, kPpTraceTiles = 256;
__device__ unsigned long long g_pp_trace[kPpTraceEvents][kPpTraceTiles];
#define PP_TRACE(ev, j)                                                                   \
  do {                                                                                    \
    if (blockIdx.x == min(7u, gridDim.x / 2) && blockIdx.y == min(3u, gridDim.y - 1) && (j) < kPpTraceTiles) \
      g_pp_trace[(ev)][(j)] = clock64();                                                  \
  } while (0)
#else
#define PP_TRACE(ev, j) \
  do {                  \
  } while (0)
#endif

namespace {

constexpr int kRows = 128;                          // query rows per tile = TMEM lanes
constexpr int kMaxQTiles = 2;                       // query tiles per CTA: QT = 2 (one CTA per SM) or 1 (two)
constexpr int kKeys = 128;                          // keys per key tile
__host__ __device__ constexpr int pp_threads(int qt) { return 32 * (4 * qt + 2); }  // softmax, producer, MMA warps
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s: only a broken pipeline waits this long
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s to let in-flight copies land on abort
constexpr float kRescaleThreshold = 8.0f;         // log2 units
constexpr int kMaxStages = 3;

// TMEM columns of tile t's S and O when a CTA holds QT tiles.
template <int QT>
__device__ __forceinline__ uint32_t col_s(int t) { return static_cast<uint32_t>(t) * 128u; }
template <int QT>
__device__ __forceinline__ uint32_t col_o(int t) { return 128u * QT + static_cast<uint32_t>(t) * 128u; }

template <int D, int QT>
struct PpCfg {
  static constexpr int ATOM = (D % 64 == 0) ? 64 : ((D % 32 == 0) ? 32 : 16);  // elements per swizzle row
  static constexpr int NATOM = D / ATOM;
  static constexpr int ROWB = ATOM * 2;                  // bytes per row of one atom block
  static constexpr uint32_t SBO = 8 * ROWB;              // 8-row core-matrix group stride
  static constexpr uint32_t LAYOUT = (ATOM == 64) ? 2u : ((ATOM == 32) ? 4u : 6u);
  static constexpr int BLOCK_BYTES = 128 * ROWB;         // one atom-column block of a 128-row tile
  static constexpr int TILE_BYTES = 128 * D * 2;         // a Q, K or V tile: NATOM blocks
  static constexpr int KSTEPS = ATOM / 16;
  // One-tile CTAs stage each softmax warp's output rows, half a row at a time,
  // so that its global stores run along rows (16-byte chunks; a padded stride
  // when a half row is an even number of chunks, against bank conflicts).
  static constexpr int STG_STRIDE = (D / 16) % 2 ? D : D + 16;
  static constexpr int STG_BYTES = QT == 1 ? 4 * 32 * STG_STRIDE : 0;
  static constexpr int FIXED = QT * TILE_BYTES + STG_BYTES + 1024 + 2048;  // Q, staging, base alignment, barriers
  // Shared memory per CTA: all of it (227 KB) for one CTA per SM; for two,
  // half of the SM's 228 KB less the 1 KB the hardware reserves per CTA.
  static constexpr int BUDGET = QT == 2 ? 232448 : 115712;
  static constexpr int STAGES = FIXED + 6 * TILE_BYTES <= BUDGET ? 3 : 2;  // K and V ring depth
  static constexpr int SMEM_BYTES = FIXED + 2 * STAGES * TILE_BYTES;
};

struct PpBars {
  uint64_t q_full, q_empty;  // Q tiles landed; the last S of the item that read them done
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[kMaxQTiles], o_full[kMaxQTiles];
  uint64_t p_half[kMaxQTiles], p_full[kMaxQTiles];  // first 64 keys of P stored; all of P stored
  uint64_t o_free[kMaxQTiles];  // the epilogue has read O (one arrival per softmax warp)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PpBars) <= 2048, "barrier block outgrew its shared-memory reservation");

struct PpParams {
  CUtensorMap tm_q, tm_k, tm_v;   // boxes of 128 rows
  AttnOut out;
  float* lse;                     // optional [head][batch][tokens], natural log
  int64_t lse_ext;                // its elements (bounds-checking builds)
  int32_t tokens, batch, n_heads, kv_tokens;
  int32_t kv_group, q_head_base, kv_head_base;  // k/v head of query head h: (q_head_base + h) / kv_group - kv_head_base
  float scale_log2;
  int32_t n_qgroups, n_kvblocks;
  int32_t n_items;                           // (query-tile group, batch, head) items of the launch
  int32_t q_start[USP_MAX_WORLD + 1];
  int32_t q_pair_prefix[USP_MAX_WORLD + 1];  // query-tile groups before query group g
  int32_t kv_start[USP_MAX_WORLD + 1];
  uint16_t heads[USP_MAX_HEADS];
};

// Key tile j of query group g: blocks in ring order g, g-1, ... (mod
// n_kvblocks), each cut into tiles of kKeys keys, the last one ragged.
struct KeyTile {
  int key0;
  int valid;
};

__device__ __forceinline__ KeyTile key_tile(const PpParams& p, int g, int j) {
  const int nb = p.n_kvblocks;
  int blk = g % nb;
  for (int s = 0; s < nb; ++s) {
    const int len = p.kv_start[blk + 1] - p.kv_start[blk];
    const int nt = (len + kKeys - 1) / kKeys;
    if (j < nt) return KeyTile{p.kv_start[blk] + j * kKeys, len - j * kKeys};
    j -= nt;
    blk = blk == 0 ? nb - 1 : blk - 1;
  }
  return KeyTile{0, 0};  // not reached for j < the group's tile count
}

// Work item `it` of a launch: query-tile group x (QT tiles of 128 rows) of one
// (batch, head), x fastest, so that CTAs running at the same time share K and V.
struct PpItem {
  int b, hm, hk, g, row0, q_end;
};
__device__ __forceinline__ PpItem pp_item(const PpParams& p, int it, int qt, bool ring) {
  const int nx = p.q_pair_prefix[p.n_qgroups];
  const int bh = it / nx;
  const int x = it - bh * nx;
  const int hi = bh / p.batch;
  PpItem w;
  w.b = bh - hi * p.batch;
  w.hm = p.heads[hi];
  w.hk = (p.q_head_base + w.hm) / p.kv_group - p.kv_head_base;  // grouped-query attention
  w.g = 0;                                                       // query group (ring)
  if (ring)
    while (w.g + 1 < p.n_qgroups && x >= p.q_pair_prefix[w.g + 1]) ++w.g;
  w.row0 = ring ? p.q_start[w.g] + (x - p.q_pair_prefix[w.g]) * (qt * kRows) : x * (qt * kRows);
  w.q_end = ring ? min(p.q_start[w.g + 1], p.tokens) : p.tokens;  // rows beyond are computed but not stored
  return w;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool bf16) {
  return bf16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

template <int D, int QT, bool BF16, bool RING>
__global__ void __launch_bounds__(pp_threads(QT), 3 - QT) attn_pp_kernel(const __grid_constant__ PpParams p) {
  using C = PpCfg<D, QT>;
  constexpr int kProducerWarp = 4 * QT;
  constexpr int kMmaWarp = 4 * QT + 1;
  constexpr uint32_t kTmemCols = 256 * QT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                    // QT tiles
  uint8_t* sK = sQ + QT * C::TILE_BYTES;                 // STAGES tiles
  uint8_t* sV = sK + C::STAGES * C::TILE_BYTES;          // STAGES tiles
  uint8_t* sStg = sV + C::STAGES * C::TILE_BYTES;        // output staging (one-tile CTAs)
  PpBars* bars = reinterpret_cast<PpBars*>(sStg + C::STG_BYTES);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = p.tokens;  // query rows; the plain kernel also takes them as keys
  // Key tiles per item (every item walks all keys). A CTA takes items
  // blockIdx.x, blockIdx.x + gridDim.x, ...; tile j of its k-th item is its
  // (k * ntiles + j)-th, which fixes every ring stage and barrier phase.
  const int ntiles = [&]() {
    if constexpr (RING) {
      int n = 0;
      for (int k = 0; k < p.n_kvblocks; ++k) n += (p.kv_start[k + 1] - p.kv_start[k] + kKeys - 1) / kKeys;
      return n;
    }
    return (T + kKeys - 1) / kKeys;
  }();
  // Two-tile CTAs take exactly one item (k = 0 below, known to the compiler).
  const int it0 = blockIdx.x, it_step = gridDim.x;
  const int it_end = QT == 2 ? min(it0 + 1, p.n_items) : p.n_items;

  // One-tile CTAs trace their start-up and epilogues in the second tile's slots.
  if (QT == 1 && threadIdx.x == 0) PP_TRACE(9, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_half[t], 128);
      mbar_init(&bars->p_full[t], 128);
      mbar_init(&bars->o_full[t], 1);
      mbar_init(&bars->o_free[t], 4);
    }
    mbar_init(&bars->drain, 1);
    // An earlier launch or CTA recorded an error: this CTA does no work.
    bars->abort = (*reinterpret_cast<volatile uint32_t*>(&g_pp_error) != 0) ? 1 : 0;
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
  if (QT == 1 && threadIdx.x == 0) PP_TRACE(10, 0);

  if (skip) {
    // fall through to the common exit
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      int nk = 0, nv = 0, nq = 0;  // K tiles, V tiles and Q groups issued, over all items
      // K (or V) of tile j of item w: the n-th tile of the CTA goes to stage
      // n % STAGES once the products that read tile n - STAGES are done.
      auto load_kv = [&](bool v, const PpItem& w, int j) -> bool {
        int& n = v ? nv : nk;
        const int st = n % C::STAGES;
        uint64_t* full = v ? &bars->v_full[st] : &bars->k_full[st];
        uint64_t* empty = v ? &bars->v_empty[st] : &bars->k_empty[st];
        if (n >= C::STAGES &&
            !mbar_wait(empty, ((n / C::STAGES) - 1) & 1, abort_flag, &g_pp_error, 40 + v, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(full, C::TILE_BYTES);
        const int key0 = RING ? key_tile(p, w.g, j).key0 : j * kKeys;
        uint8_t* dst = (v ? sV : sK) + st * C::TILE_BYTES;
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(v ? &p.tm_v : &p.tm_k, full, dst + a * C::BLOCK_BYTES, a * C::ATOM, w.hk, key0, w.b);
        ++n;
        return true;
      };
      bool go = true;
      for (int it = it0, k = 0; go && it < it_end; it += it_step, ++k) {
        if constexpr (QT == 2) k = 0;
        const PpItem w = pp_item(p, it, QT, RING);
        go = load_kv(false, w, 0);
        // Q of this item once the last S of the previous one (which read Q) is done.
        if (go && k > 0)
          go = mbar_wait(&bars->q_empty, (k - 1) & 1, abort_flag, &g_pp_error, 39, kWaitLimitNs);
        if (go) {
          mbar_arrive_expect_tx(&bars->q_full, QT * C::TILE_BYTES);
          for (int t = 0; t < QT; ++t)
            for (int a = 0; a < C::NATOM; ++a)
              tma_load_4d(&p.tm_q, &bars->q_full, sQ + t * C::TILE_BYTES + a * C::BLOCK_BYTES, a * C::ATOM, w.hm,
                          w.row0 + t * kRows, w.b);
          ++nq;
        }
        // Issue order follows consumption: K(0), then K(j+1) before V(j).
        for (int j = 0; go && j < ntiles; ++j) {
          if (j + 1 < ntiles) go = load_kv(false, w, j + 1);
          if (go) go = load_kv(true, w, j);
        }
      }
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        for (int j = (nk > C::STAGES ? nk - C::STAGES : 0); j < nk; ++j)
          mbar_wait_drain(&bars->k_full[j % C::STAGES], (j / C::STAGES) & 1, kDrainLimitNs);
        for (int j = (nv > C::STAGES ? nv - C::STAGES : 0); j < nv; ++j)
          mbar_wait_drain(&bars->v_full[j % C::STAGES], (j / C::STAGES) & 1, kDrainLimitNs);
        if (nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1, kDrainLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_f16(kRows, kKeys, BF16, false);
      const uint32_t idesc_pv = make_idesc_f16(kRows, D, BF16, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      // S_t = Q_t K^T for the K tile in ring stage st (already landed).
      auto issue_s = [&](int t, int st, int jg) {
        PP_TRACE(t, jg);
#pragma unroll
        for (int a = 0; a < C::NATOM; ++a)
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            const uint64_t adesc =
                make_smem_desc(q_addr + t * C::TILE_BYTES + a * C::BLOCK_BYTES + ks * 32, 16, C::SBO, C::LAYOUT);
            const uint64_t bdesc =
                make_smem_desc(k_addr + st * C::TILE_BYTES + a * C::BLOCK_BYTES + ks * 32, 16, C::SBO, C::LAYOUT);
            umma_ss(tmem + col_s<QT>(t), adesc, bdesc, idesc_qk, (a > 0 || ks > 0) ? 1u : 0u);
          }
        umma_commit(&bars->s_full[t]);
        if (QT == 1) PP_TRACE(15, jg);
      };
      // O_t += P_t V for the CTA's tile jg (tile j of its item): the products
      // over the first 64 keys once the softmax of tile t has stored that half
      // of P_t, the rest once it has stored all of it. Before an item's first
      // P V, the epilogue of the CTA's previous item (k - 1) must have read O_t.
      auto issue_pv = [&](int t, int j, int jg, int k, int st) -> bool {
        if (j == 0 && k > 0 &&
            !mbar_wait(&bars->o_free[t], (k - 1) & 1, abort_flag, &g_pp_error, 56 + t, kWaitLimitNs))
          return false;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(h == 0 ? &bars->p_half[t] : &bars->p_full[t], jg & 1, abort_flag, &g_pp_error,
                         h == 0 ? 58 + t : 43 + t, kWaitLimitNs))
            return false;
          if (h == 0) PP_TRACE(2 + t, jg);
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
            const uint64_t bdesc =
                make_smem_desc(v_addr + st * C::TILE_BYTES + kk * 16 * C::ROWB, C::BLOCK_BYTES, C::SBO, C::LAYOUT);
            umma_ts(tmem + col_o<QT>(t), tmem + col_s<QT>(t) + kk * 8, bdesc, idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        return true;
      };
      auto wait_k = [&](int jg) {
        const int st = jg % C::STAGES;
        const bool r = mbar_wait(&bars->k_full[st], (jg / C::STAGES) & 1, abort_flag, &g_pp_error, 45, kWaitLimitNs);
        tc_fence_after();
        return r;
      };
      auto wait_v = [&](int jg) {
        const int st = jg % C::STAGES;
        const bool r = mbar_wait(&bars->v_full[st], (jg / C::STAGES) & 1, abort_flag, &g_pp_error, 46, kWaitLimitNs);
        tc_fence_after();
        return r;
      };
      bool ok = true;
      for (int it = it0, k = 0; ok && it < it_end; it += it_step, ++k) {
        if constexpr (QT == 2) k = 0;
        const int base = k * ntiles;  // the CTA's tile index of this item's tile 0
        ok = mbar_wait(&bars->q_full, k & 1, abort_flag, &g_pp_error, 42, kWaitLimitNs);
        tc_fence_after();
        if (QT == 1) PP_TRACE(11, k);
        if (ok) ok = wait_k(base);
        if (QT == 1) PP_TRACE(14, k);
        if (!ok) break;
        // S_t(0) overwrites P_t of the previous item, whose P V was issued before.
        issue_s(0, base % C::STAGES, base);
        if constexpr (QT == 2) issue_s(1, base % C::STAGES, base);
        umma_commit(&bars->k_empty[base % C::STAGES]);
        for (int j = 1; ok && j < ntiles; ++j) {
          const int vs = (base + j - 1) % C::STAGES;
          if (!(ok = wait_v(base + j - 1))) break;
          if (!(ok = issue_pv(0, j - 1, base + j - 1, k, vs))) break;
          if (!(ok = wait_k(base + j))) break;
          const int ks = (base + j) % C::STAGES;
          issue_s(0, ks, base + j);  // after P_A(j-1) V: S_A(j) overwrites P_A(j-1)
          if constexpr (QT == 2) {
            if (!(ok = issue_pv(1, j - 1, base + j - 1, k, vs))) break;
            umma_commit(&bars->v_empty[vs]);
            issue_s(1, ks, base + j);
          } else {
            umma_commit(&bars->v_empty[vs]);
          }
          umma_commit(&bars->k_empty[ks]);
        }
        if (!ok) break;
        umma_commit(&bars->q_empty);  // every S of this item issued: Q may be replaced once they are done
        const int j = ntiles - 1, jg = base + j, vs = jg % C::STAGES;
        ok = wait_v(jg);
        if (ok) ok = issue_pv(0, j, jg, k, vs);
        if (ok) umma_commit(&bars->o_full[0]);
        if constexpr (QT == 2) {
          if (ok) ok = issue_pv(1, j, jg, k, vs);
          if (ok) umma_commit(&bars->o_full[1]);
        }
        if (ok) umma_commit(&bars->v_empty[vs]);
      }
      // All MMAs this thread issued must finish before TMEM is released.
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;                         // query tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;             // TMEM lane = query row in the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t sc = lane_addr + col_s<QT>(t);
    const uint32_t oc = lane_addr + col_o<QT>(t);
    const float sl2 = p.scale_log2;
    const bool tr0 = quarter == 0 && lane == 0;
    // Epilogue of the CTA's k-th item `it` (running maximum m, denominator l):
    // O of this tile, normalised, to the rows' destinations. Returns false if
    // a wait gave up.
    auto epilogue = [&](int it, int k, float m, float l) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full[t], k & 1, abort_flag, &g_pp_error, 52 + t,
                                             kWaitLimitNs)))
        return false;
      tc_fence_after();
      if (QT == 1 && tr0) PP_TRACE(12, k);
      // The whole row of O in one round of TMEM loads; then O may be overwritten.
      uint32_t o[D];
#pragma unroll
      for (int c = 0; c < D / 16; ++c) tmem_ld16(oc + c * 16, *reinterpret_cast<uint32_t(*)[16]>(o + c * 16));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free[t]);
      const float inv_l = 1.f / l;
      const PpItem w = pp_item(p, it, QT, RING);
      const int tr = w.row0 + t * kRows + row;  // row of the full sequence
      const bool row_ok = tr < w.q_end;
      if (p.lse != nullptr && row_ok) {  // sum_j exp(scale s_j) = 2^m * l
        const int64_t li = (static_cast<int64_t>(w.hm) * p.batch + w.b) * T + tr;
        if (in_bounds(li, 1, p.lse_ext, 22, &g_pp_bounds)) p.lse[li] = (m + log2f(l)) * 0.69314718055994531f;
      }
      const AttnOut& out = p.out;
      int seg_lo = 0, seg_hi = 0;
      int64_t row_in_seg = 0;
      if (row_ok) {
        if (tr < out.prefix) {  // a replicated prefix row goes to every segment
          seg_lo = 0;
          seg_hi = out.nseg;
          row_in_seg = tr;
        } else {
          const int64_t tok = tr - out.prefix;
          int sg = 0;
          while (sg + 1 < out.nseg && tok >= out.seg_start[sg + 1]) ++sg;
          seg_lo = sg;
          seg_hi = sg + 1;
          row_in_seg = out.prefix + tok - out.seg_start[sg];
        }
      }
#pragma unroll
      for (int i = 0; i < D / 2; ++i)
        o[i] = pack2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l, BF16);
      // This row's destination in segment sg (null: out of range).
      auto row_dst = [&](int sg) -> uint16_t* {
        const int64_t rows_s = out.prefix + out.seg_len[sg];
        const int64_t elem =
            ((static_cast<int64_t>(w.b) * rows_s + row_in_seg) * out.out_heads + w.hm - out.head_base) * D;
        if (!in_bounds(elem, D, static_cast<int64_t>(p.batch) * rows_s * out.out_heads * D, 23, &g_pp_bounds))
          return nullptr;
        return static_cast<uint16_t*>(out.seg_ptr[sg]) + elem;
      };
      int sg_direct = seg_lo;  // segments this thread writes itself, from its registers
      if constexpr (QT == 1) {
        // The warp's 32 rows, half a row per round, through its staging block:
        // each thread writes its half row, then the warp stores the block in
        // row-major order, consecutive threads writing consecutive 16-byte
        // chunks of a row. The first segment goes this way; a replicated
        // prefix row's other segments are written directly below.
        constexpr int CH = D / 16;  // 16-byte chunks per half row
        const uint64_t my_dst = row_ok ? reinterpret_cast<uint64_t>(row_dst(seg_lo)) : 0;
        const uint32_t stg = smem_u32(sStg) + quarter * (32 * C::STG_STRIDE);
        sg_direct = seg_lo + 1;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const int i = h * (D / 4) + 4 * c;
            st_shared_v4(stg + lane * C::STG_STRIDE + c * 16, o[i], o[i + 1], o[i + 2], o[i + 3]);
          }
          __syncwarp();
#pragma unroll
          for (int st = 0; st < CH; ++st) {
            const int q = st * 32 + lane;  // chunk q of the block: row q / CH, chunk q % CH
            const int r = q / CH, c = q - r * CH;
            const uint4 v = ld_shared_v4(stg + r * C::STG_STRIDE + c * 16);
            const uint64_t d = __shfl_sync(0xffffffffu, my_dst, r);
            if (d != 0) reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(d) + h * (D / 2))[c] = v;
          }
          __syncwarp();
        }
      }
      for (int sg = sg_direct; sg < seg_hi; ++sg) {
        uint4* dst = reinterpret_cast<uint4*>(row_dst(sg));
        if (dst == nullptr) continue;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      }
      if (QT == 1 && tr0) PP_TRACE(13, k);
      return true;
    };
    bool ok = true;
    for (int it = it0, k = 0; ok && it < it_end; it += it_step, ++k) {
      if constexpr (QT == 2) k = 0;
      int kb_blk = 0, kb_left = 0;
      if constexpr (RING) {
        kb_blk = pp_item(p, it, QT, RING).g % p.n_kvblocks;
        kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
      }
      float m = -INFINITY;  // running maximum, log2 domain
      float l = 0.f;        // running denominator
      for (int j = 0; j < ntiles; ++j) {
        const int jg = k * ntiles + j;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], jg & 1, abort_flag, &g_pp_error, 50 + t,
                                               kWaitLimitNs))) {
          ok = false;
          break;
        }
        if (tr0) PP_TRACE(4 + 5 * t, jg);
        tc_fence_after();
        uint32_t sr[kKeys];
#pragma unroll
        for (int c = 0; c < kKeys; c += 32) tmem_ld32(sc + c, sr + c);
        tmem_wait_ld();
        if (tr0) PP_TRACE(5 + 5 * t, jg);
        float* s = reinterpret_cast<float*>(sr);
        const int valid = RING ? kb_left : T - j * kKeys;  // valid keys of this tile (>= kKeys: all)
        if (valid < kKeys) {
#pragma unroll
          for (int c = 0; c < kKeys; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        // Row maximum: eight independent three-input chains, then a tree.
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float a = fmaxf(s[i], s[i + 8]);
#pragma unroll
          for (int c = i + 16; c < kKeys; c += 16) a = max3(a, s[c], s[c + 8]);
          mx8[i] = a;
        }
        const float mx = max3(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_new = fmaxf(m, mx * sl2);
        if (tr0) PP_TRACE(6 + 5 * t, jg);
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
          // O holds sum_{i<j} exp2(s_i - m) v_i (its last P V completed before
          // this tile's S did); bring it to the new maximum.
          const float alpha = ex2_approx(m - m_new);
          m = m_new;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(oc + c * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(oc + c * 16, o);
          }
          tmem_wait_st();
        }
        // p = 2^(s*scale*log2e - m), packed to the input type, written over the
        // first 64 columns of S (already in registers) in two halves. Masked
        // entries (s = -inf) give exactly 0.
        // The scaling and the row sum run on packed fp32 pairs (one instruction
        // per two values). Measured and not kept: rounding P on the integer pipe
        // instead of cvt (10% slower); a quarter or half of the exponentials as a
        // degree-3 polynomial on the FMA pipe (4-5% slower).
        const uint64_t scale2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-m, -m);
        uint64_t acc2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[64 * h + c], s[64 * h + c + 1]), scale2, negm2), x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            acc2[(c >> 1) & 3] = f2_add(acc2[(c >> 1) & 3], f2_pack(p0, p1));
            pk[c / 2] = pack2(p0, p1, BF16);
          }
          tmem_st32(sc + 32 * h, pk);
          if (h == 0) {
            // The products over these 64 keys may start while the rest is computed.
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_half[t]);
          }
        }
        float a0, a1, a2, a3, a4, a5, a6, a7;
        f2_unpack(acc2[0], a0, a1);
        f2_unpack(acc2[1], a2, a3);
        f2_unpack(acc2[2], a4, a5);
        f2_unpack(acc2[3], a6, a7);
        l += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
        if (tr0) PP_TRACE(7 + 5 * t, jg);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[t]);
        if (tr0) PP_TRACE(8 + 5 * t, jg);
        if constexpr (RING) {
          kb_left -= kKeys;
          if (kb_left <= 0) {
            kb_blk = kb_blk == 0 ? p.n_kvblocks - 1 : kb_blk - 1;
            kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
          }
        }
      }
      if (!ok) break;
      ok = epilogue(it, k, m, l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int QT, bool BF16>
int launch_pp_d(const AttnLaunch& L, cudaStream_t stream) {
  using C = PpCfg<D, QT>;
  static_assert(C::SMEM_BYTES <= C::BUDGET, "shared memory above the per-CTA budget");
  // Two CTAs per SM need the largest shared-memory carveout.
  for (auto* fn : {attn_pp_kernel<D, QT, BF16, false>, attn_pp_kernel<D, QT, BF16, true>})
    if (int rc = ensure_smem_limit(reinterpret_cast<const void*>(fn), C::SMEM_BYTES,
                                   "cudaFuncSetAttribute(attention smem)", QT == 1 ? 100 : -1))
      return rc;
  thread_local PpParams p;
  memset(&p, 0, sizeof(p));
  int rc;
  const int kv_tokens = L.kv_tokens > 0 ? L.kv_tokens : L.tokens;
  const bool ring = L.blocks.n_qgroups > 0 || L.blocks.n_kvblocks > 0;
  if (!ring && kv_tokens != L.tokens)
    return set_error(USP_ERR_INVALID_ARG, "internal: the plain attention kernel takes as many keys as queries");
  if ((rc = make_map(&p.tm_q, L.in.q, L.in.qv, L, L.tokens, C::ATOM, kRows)) != USP_OK) return rc;
  if ((rc = make_map(&p.tm_k, L.in.k, L.in.kvv, L, kv_tokens, C::ATOM, kKeys)) != USP_OK) return rc;
  if ((rc = make_map(&p.tm_v, L.in.v, L.in.kvv, L, kv_tokens, C::ATOM, kKeys)) != USP_OK) return rc;
  if (!fill_blocks(L, kv_tokens, QT * kRows, p.n_qgroups, p.n_kvblocks, p.q_start, p.q_pair_prefix, p.kv_start))
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
  const int64_t items = static_cast<int64_t>(p.q_pair_prefix[p.n_qgroups]) * L.batch * L.n_heads;
  if (items > INT32_MAX) return set_error(USP_ERR_UNSUPPORTED, "attention: %lld query tiles in one launch", (long long)items);
  p.n_items = static_cast<int32_t>(items);
  // Two query tiles: one CTA per item. One query tile: two CTAs per SM (or
  // the caller's cap) walk the items, each starting an item's loads and first
  // Q K^T under the end of the one before.
  const int64_t walkers = L.max_ctas > 0 ? L.max_ctas : 2 * static_cast<int64_t>(sm_count());
  const int64_t ctas = QT == 2 ? items : std::min<int64_t>(items, walkers);
  const dim3 grid(static_cast<unsigned>(ctas));
  if (ring)
    attn_pp_kernel<D, QT, BF16, true><<<grid, pp_threads(QT), C::SMEM_BYTES, stream>>>(p);
  else
    attn_pp_kernel<D, QT, BF16, false><<<grid, pp_threads(QT), C::SMEM_BYTES, stream>>>(p);
  count_launch();
  return cuda_check(cudaGetLastError(), "attention (tcgen05, 128-key tiles) launch");
}

template <bool BF16>
int launch_pp_dtype(const AttnLaunch& L, cudaStream_t stream) {
  if (L.kernel == USP_ATTN_TWO_CTA) {
    switch (L.head_dim) {
      case 64: return launch_pp_d<64, 1, BF16>(L, stream);
      case 80: return launch_pp_d<80, 1, BF16>(L, stream);
      default: return set_error(USP_ERR_UNSUPPORTED, "two-CTA attention: head_dim %d not built", L.head_dim);
    }
  }
  switch (L.head_dim) {
    case 64: return launch_pp_d<64, 2, BF16>(L, stream);
    case 80: return launch_pp_d<80, 2, BF16>(L, stream);
    case 96: return launch_pp_d<96, 2, BF16>(L, stream);
    case 112: return launch_pp_d<112, 2, BF16>(L, stream);
    case 128: return launch_pp_d<128, 2, BF16>(L, stream);
    default: return set_error(USP_ERR_UNSUPPORTED, "two-tile attention: head_dim %d not built", L.head_dim);
  }
}

}  // namespace

bool attention_pp_supported(int dtype, int head_dim, int kernel) {
  if (dtype != USP_BF16 && dtype != USP_FP16) return false;
  if (kernel == USP_ATTN_TWO_CTA) return head_dim == 64 || head_dim == 80;
  return head_dim % 16 == 0 && head_dim >= 64 && head_dim <= 128;
}

int launch_attention_pp(const AttnLaunch& L, cudaStream_t stream) {
  if (L.n_heads == 0 || L.batch == 0 || L.tokens == 0) return USP_OK;
  return L.dtype == USP_BF16 ? launch_pp_dtype<true>(L, stream) : launch_pp_dtype<false>(L, stream);
}

int read_pp_error(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_pp_error, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read device error word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_pp_error, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset device error word");
  }
  return USP_OK;
}

#ifdef USP_TRACE
extern "C" int usp_debug_read_trace_pp(unsigned long long* out, int n) {
  const int total = kPpTraceEvents * kPpTraceTiles;
  if (n > total) n = total;
  return cudaMemcpyFromSymbol(out, g_pp_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 5;
}
#endif

int read_pp_bounds(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_pp_bounds, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read two-tile attention bounds word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_pp_bounds, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset two-tile attention bounds word");
  }
  return USP_OK;
}

}  // namespace usp
