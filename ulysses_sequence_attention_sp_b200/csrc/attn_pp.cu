// Non-causal softmax attention on the tcgen05 tensor cores, two query tiles
// per CTA ("ping-pong").
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
// How it is organised differs. One CTA takes two 128-row query tiles A and B
// of one (batch, head) and walks the keys in tiles of 128:
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: one thread
//               per query row (TMEM lane = row), holding the row's 128 scores,
//               so no partial maxima are exchanged between threads
//   warp 8      TMA producer: Q_A and Q_B once, then K and V tiles into rings
//   warp 9      TMEM allocator and MMA issuer (one thread), in the order
//                 S_A(0) S_B(0) | PV_A(j-1) S_A(j) PV_B(j-1) S_B(j) | ...
//               so that while the softmax of one tile runs, the tensor core
//               works on the other tile's products.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [384,384+D).
// P (128 keys, two 16-bit values per column) is written over the first 64
// columns of its tile's S, which the softmax has already read into registers;
// the next S of that tile is issued only after the P.V that reads P, and the
// tensor core runs one thread's MMAs in issue order.
// O is rescaled in TMEM only when a row maximum grows by more than 2^8 (the
// stale maximum is kept otherwise: exact, since numerator and denominator use
// the same maximum). A tile's O is only ever written by its own P.V, which
// has completed whenever the tile's next S has (one commit covers both).
#include <cmath>

#include "device_common.cuh"
#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_pp_error;   // first wait that ran out (site code), 0 if none
__device__ uint32_t g_pp_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

// Pipeline trace (built only with -DUSP_TRACE): clock64() at pipeline events
// of CTA 7, [event][key tile]; read with usp_debug_read_trace_pp.
#ifdef USP_TRACE
constexpr int kPpTraceEvents = 16, kPpTraceTiles = 256;
__device__ unsigned long long g_pp_trace[kPpTraceEvents][kPpTraceTiles];
#define PP_TRACE(ev, j)                                                                   \
  do {                                                                                    \
    if (blockIdx.x == 7 && blockIdx.y == 0 && (j) < kPpTraceTiles) g_pp_trace[(ev)][(j)] = clock64(); \
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
  static constexpr int FIXED = QT * TILE_BYTES + 1024 + 2048;  // Q tiles, base alignment, barriers
  // Shared memory per CTA: all of it (227 KB) for one CTA per SM; for two,
  // half of the SM's 228 KB less the 1 KB the hardware reserves per CTA.
  static constexpr int BUDGET = QT == 2 ? 232448 : 115712;
  static constexpr int STAGES = FIXED + 6 * TILE_BYTES <= BUDGET ? 3 : 2;  // K and V ring depth
  static constexpr int SMEM_BYTES = FIXED + 2 * STAGES * TILE_BYTES;
};

struct PpBars {
  uint64_t q_full;
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[kMaxQTiles], p_full[kMaxQTiles], o_full[kMaxQTiles];
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
  int32_t q_start[USP_MAX_WORLD + 1];
  int32_t q_pair_prefix[USP_MAX_WORLD + 1];  // CTAs (query-tile pairs) before group g
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
  PpBars* bars = reinterpret_cast<PpBars*>(sV + C::STAGES * C::TILE_BYTES);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int hi = blockIdx.y / p.batch;
  const int b = blockIdx.y - hi * p.batch;
  const int hm = p.heads[hi];
  const int hk = (p.q_head_base + hm) / p.kv_group - p.kv_head_base;  // grouped-query attention
  const int T = p.tokens;  // query rows; the plain kernel also takes them as keys
  int g = 0;               // query group (ring), and the CTA's first query row
  if constexpr (RING)
    while (g + 1 < p.n_qgroups && static_cast<int>(blockIdx.x) >= p.q_pair_prefix[g + 1]) ++g;
  const int row0 = RING ? p.q_start[g] + (static_cast<int>(blockIdx.x) - p.q_pair_prefix[g]) * (QT * kRows)
                        : static_cast<int>(blockIdx.x) * (QT * kRows);
  const int q_end = RING ? min(p.q_start[g + 1], T) : T;  // rows beyond are computed but not stored
  const int ntiles = [&]() {
    if constexpr (RING) {
      int n = 0;
      for (int k = 0; k < p.n_kvblocks; ++k) n += (p.kv_start[k + 1] - p.kv_start[k] + kKeys - 1) / kKeys;
      return n;
    }
    return (T + kKeys - 1) / kKeys;
  }();

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 128);
      mbar_init(&bars->o_full[t], 1);
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

  if (skip) {
    // fall through to the common exit
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      mbar_arrive_expect_tx(&bars->q_full, QT * C::TILE_BYTES);
      for (int t = 0; t < QT; ++t)
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_q, &bars->q_full, sQ + t * C::TILE_BYTES + a * C::BLOCK_BYTES, a * C::ATOM, hm,
                      row0 + t * kRows, b);
      auto key0_of = [&](int j) { return RING ? key_tile(p, g, j).key0 : j * kKeys; };
      // K of tile j into stage j % STAGES once the S products of tile j - STAGES are done.
      auto load_k = [&](int j) -> bool {
        const int st = j % C::STAGES;
        if (j >= C::STAGES &&
            !mbar_wait(&bars->k_empty[st], ((j / C::STAGES) - 1) & 1, abort_flag, &g_pp_error, 40, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->k_full[st], C::TILE_BYTES);
        const int key0 = key0_of(j);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_k, &bars->k_full[st], sK + st * C::TILE_BYTES + a * C::BLOCK_BYTES, a * C::ATOM, hk,
                      key0, b);
        return true;
      };
      // V of tile j once the P V products of tile j - STAGES are done.
      auto load_v = [&](int j) -> bool {
        const int st = j % C::STAGES;
        if (j >= C::STAGES &&
            !mbar_wait(&bars->v_empty[st], ((j / C::STAGES) - 1) & 1, abort_flag, &g_pp_error, 41, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
        const int key0 = key0_of(j);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_v, &bars->v_full[st], sV + st * C::TILE_BYTES + a * C::BLOCK_BYTES, a * C::ATOM, hk,
                      key0, b);
        return true;
      };
      // Issue order follows consumption: K(0), then K(j+1) before V(j).
      int nk = 0, nv = 0;
      bool go = load_k(0);
      nk += go;
      for (int j = 0; go && j < ntiles; ++j) {
        if (j + 1 < ntiles) {
          go = load_k(j + 1);
          nk += go;
        }
        if (go) {
          go = load_v(j);
          nv += go;
        }
      }
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        for (int j = (nk > C::STAGES ? nk - C::STAGES : 0); j < nk; ++j)
          mbar_wait_drain(&bars->k_full[j % C::STAGES], (j / C::STAGES) & 1, kDrainLimitNs);
        for (int j = (nv > C::STAGES ? nv - C::STAGES : 0); j < nv; ++j)
          mbar_wait_drain(&bars->v_full[j % C::STAGES], (j / C::STAGES) & 1, kDrainLimitNs);
        mbar_wait_drain(&bars->q_full, 0, kDrainLimitNs);
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
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, &g_pp_error, 42, kWaitLimitNs);
      tc_fence_after();
      // S_t = Q_t K^T for the K tile in ring stage st (already landed).
#ifdef USP_TRACE
      int s_count[2] = {0, 0};
#endif
      auto issue_s = [&](int t, int st) {
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
#ifdef USP_TRACE
        const int si = s_count[t]++;
        PP_TRACE(t, si);
#endif
      };
      // O_t += P_t(j) V_j once the softmax of tile t has stored P_t(j) (V stage st landed).
      auto issue_pv = [&](int t, int j, int st) -> bool {
        if (!mbar_wait(&bars->p_full[t], j & 1, abort_flag, &g_pp_error, 43 + t, kWaitLimitNs)) return false;
        PP_TRACE(2 + t, j);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint64_t bdesc =
              make_smem_desc(v_addr + st * C::TILE_BYTES + kk * 16 * C::ROWB, C::BLOCK_BYTES, C::SBO, C::LAYOUT);
          umma_ts(tmem + col_o<QT>(t), tmem + col_s<QT>(t) + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        return true;
      };
      auto wait_k = [&](int j) {
        const int st = j % C::STAGES;
        const bool r = mbar_wait(&bars->k_full[st], (j / C::STAGES) & 1, abort_flag, &g_pp_error, 45, kWaitLimitNs);
        tc_fence_after();
        return r;
      };
      auto wait_v = [&](int j) {
        const int st = j % C::STAGES;
        const bool r = mbar_wait(&bars->v_full[st], (j / C::STAGES) & 1, abort_flag, &g_pp_error, 46, kWaitLimitNs);
        tc_fence_after();
        return r;
      };
      if (ok) ok = wait_k(0);
      if (ok) {
        issue_s(0, 0);
        if constexpr (QT == 2) issue_s(1, 0);
        umma_commit(&bars->k_empty[0]);
      }
      for (int j = 1; ok && j < ntiles; ++j) {
        const int vs = (j - 1) % C::STAGES;
        if (!(ok = wait_v(j - 1))) break;
        if (!(ok = issue_pv(0, j - 1, vs))) break;
        if (!(ok = wait_k(j))) break;
        const int ks = j % C::STAGES;
        issue_s(0, ks);  // after P_A(j-1) V: S_A(j) overwrites P_A(j-1)
        if constexpr (QT == 2) {
          if (!(ok = issue_pv(1, j - 1, vs))) break;
          umma_commit(&bars->v_empty[vs]);
          issue_s(1, ks);
        } else {
          umma_commit(&bars->v_empty[vs]);
        }
        umma_commit(&bars->k_empty[ks]);
      }
      if (ok) {
        const int j = ntiles - 1, vs = j % C::STAGES;
        ok = wait_v(j);
        if (ok) ok = issue_pv(0, j, vs);
        if (ok) umma_commit(&bars->o_full[0]);
        if constexpr (QT == 2) {
          if (ok) ok = issue_pv(1, j, vs);
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
    int kb_blk = 0, kb_left = 0;
    if constexpr (RING) {
      kb_blk = g % p.n_kvblocks;
      kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
    }
    float m = -INFINITY;  // running maximum, log2 domain
    float l = 0.f;        // running denominator
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], j & 1, abort_flag, &g_pp_error, 50 + t,
                                             kWaitLimitNs))) {
        ok = false;
        break;
      }
      const bool tr0 = (warp & 3) == 0 && lane == 0;
      if (tr0) PP_TRACE(4 + 5 * t, j);
      tc_fence_after();
      uint32_t sr[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys; c += 32) tmem_ld32(sc + c, sr + c);
      tmem_wait_ld();
      if (tr0) PP_TRACE(5 + 5 * t, j);
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
      if (tr0) PP_TRACE(6 + 5 * t, j);
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
      }
      float a0, a1, a2, a3, a4, a5, a6, a7;
      f2_unpack(acc2[0], a0, a1);
      f2_unpack(acc2[1], a2, a3);
      f2_unpack(acc2[2], a4, a5);
      f2_unpack(acc2[3], a6, a7);
      l += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
      if (tr0) PP_TRACE(7 + 5 * t, j);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[t]);
      if (tr0) PP_TRACE(8 + 5 * t, j);
      if constexpr (RING) {
        kb_left -= kKeys;
        if (kb_left <= 0) {
          kb_blk = kb_blk == 0 ? p.n_kvblocks - 1 : kb_blk - 1;
          kb_left = p.kv_start[kb_blk + 1] - p.kv_start[kb_blk];
        }
      }
    }
    // Epilogue: O of this tile, normalised, to the rows' destinations.
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_full[t], 0, abort_flag, &g_pp_error, 52 + t,
                                                 kWaitLimitNs))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int tr = row0 + t * kRows + row;  // row of the full sequence
      const bool row_ok = tr < q_end;
      if (p.lse != nullptr && row_ok) {  // sum_j exp(scale s_j) = 2^m * l
        const int64_t li = (static_cast<int64_t>(hm) * p.batch + b) * T + tr;
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
      for (int c = 0; c < D / 16; ++c) {
        uint32_t o[16];
        tmem_ld16(oc + c * 16, o);
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
          if (!in_bounds(elem, 16, static_cast<int64_t>(p.batch) * rows_s * out.out_heads * D, 23, &g_pp_bounds))
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
  const dim3 grid(p.q_pair_prefix[p.n_qgroups], L.batch * L.n_heads);
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
