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
// One CTA computes one 128-row query tile of one (batch, head):
//   warp 8      TMA producer: Q once, then K_j and V_j tiles into smem rings
//   warp 9      TMEM allocator and MMA issuer (one thread):
//                 S_j = Q K_j^T      (SS: both operands in smem)  -> TMEM S[j%2]
//                 O  += P_{j-1} V_{j-1} (TS: P in TMEM, V in smem) -> TMEM O
//   warps 0-7   softmax: warps w and w+4 own query rows 32(w%4).. (TMEM lane =
//               row), each taking half of the key columns of a tile; online
//               softmax in the log2 domain; O is rescaled in TMEM only when a
//               row maximum grows by more than 2^8, otherwise the stale
//               maximum is kept (exact: the final division uses the same
//               maximum for numerator and denominator).
// TMEM columns: S0 [0,128), S1 [128,256), O [256,256+D), P0 [384,448), P1 [448,512).
#include <cmath>
#include <cstdio>
#include <mutex>

#include "device_common.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_attn_error;  // first wait that ran out (site code), 0 if none

// Pipeline trace (built only with -DUSP_TRACE): clock64() at pipeline events
// of one CTA, [event][key tile]; read with usp_debug_read_trace.
#ifdef USP_TRACE
constexpr int kTraceEvents = 12, kTraceTiles = 256;
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

constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 128;  // keys per tile
constexpr int kThreads = 320;  // 8 softmax warps, TMA warp, MMA warp
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s: only a broken pipeline waits this long
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s to let in-flight copies land on abort
constexpr float kRescaleThreshold = 8.0f;          // log2 units
constexpr int kPolyEvery = 4;                      // one exp2 pair in four on the FMA pipe

template <int D>
struct Cfg {
  static constexpr int ATOM = (D % 64 == 0) ? 64 : ((D % 32 == 0) ? 32 : 16);  // elements per swizzle row
  static constexpr int NATOM = D / ATOM;
  static constexpr int ROWB = ATOM * 2;               // bytes per row of one atom block
  static constexpr int BLOCK_BYTES = kBM * ROWB;      // one atom block of a 128-row tile
  static constexpr int TILE_BYTES = kBM * D * 2;
  static constexpr uint32_t SBO = 8 * ROWB;           // 8-row core-matrix group stride
  static constexpr uint32_t LAYOUT = (ATOM == 64) ? 2u : ((ATOM == 32) ? 4u : 6u);
  static constexpr int KSTAGES = (D <= 64) ? 4 : 3;
  static constexpr int VSTAGES = (D <= 64) ? 4 : ((D <= 112) ? 3 : 2);
  // Q + KSTAGES K tiles + VSTAGES V tiles, 1 KB alignment slack, barriers
  static constexpr int SMEM_BYTES = TILE_BYTES * (1 + KSTAGES + VSTAGES) + 1024 + 2560;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2];
  uint64_t o_full, drain;
  uint64_t xbar[4];          // partial-maximum exchange between warps w and w+4
  uint32_t tmem_base;
  int abort;
  float xch[2 * 2 * kBM];    // [tile parity][half][row]
};

static_assert(sizeof(Bars) + 8 <= 2560, "barrier block outgrew its shared-memory reservation");

struct TcParams {
  CUtensorMap tm_q, tm_k, tm_v;
  AttnOut out;
  int32_t tokens, batch, n_heads, pad0;
  float scale_log2;
  uint16_t heads[USP_MAX_HEADS];
};

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool bf16) {
  return bf16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::TILE_BYTES;
  uint8_t* sV = sK + C::KSTAGES * C::TILE_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(sV + C::VSTAGES * C::TILE_BYTES);
  volatile int* abort_flag = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qtile = blockIdx.x;
  const int hi = blockIdx.y / p.batch;
  const int b = blockIdx.y - hi * p.batch;
  const int hm = p.heads[hi];
  const int T = p.tokens;
  const int ntiles = (T + kBN - 1) / kBN;
#ifdef USP_TRACE
  const bool trace_cta = blockIdx.x == 7 && blockIdx.y == 0;
#endif

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::KSTAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::VSTAGES; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], kSoftmaxThreads);
      mbar_init(&bars->p_full[i], kSoftmaxThreads);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->xbar[q], 64);
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
      mbar_arrive_expect_tx(&bars->q_full, C::TILE_BYTES);
      for (int a = 0; a < C::NATOM; ++a)
        tma_load_4d(&p.tm_q, &bars->q_full, sQ + a * C::BLOCK_BYTES, a * C::ATOM, hm, qtile * kBM, b);
      // K runs one tile ahead of V: K_{j+1} is needed (for S_{j+1}) before V_j.
      auto load_k = [&](int j) -> bool {
        const int st = j % C::KSTAGES;
        if (j >= C::KSTAGES &&
            !mbar_wait(&bars->k_empty[st], ((j / C::KSTAGES) - 1) & 1, abort_flag, &g_attn_error, 10, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->k_full[st], C::TILE_BYTES);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_k, &bars->k_full[st], sK + st * C::TILE_BYTES + a * C::BLOCK_BYTES, a * C::ATOM, hm,
                      j * kBN, b);
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j % C::VSTAGES;
        if (j >= C::VSTAGES &&
            !mbar_wait(&bars->v_empty[st], ((j / C::VSTAGES) - 1) & 1, abort_flag, &g_attn_error, 11, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
        for (int a = 0; a < C::NATOM; ++a)
          tma_load_4d(&p.tm_v, &bars->v_full[st], sV + st * C::TILE_BYTES + a * C::BLOCK_BYTES, a * C::ATOM, hm,
                      j * kBN, b);
        return true;
      };
      int nk = 0, nv = 0;  // tiles issued
      if (load_k(0)) {
        nk = 1;
        for (int j = 0; j < ntiles; ++j) {
          if (j + 1 < ntiles) {
            if (!load_k(j + 1)) break;
            nk = j + 2;
            USP_TRACE_EV(0, j + 1);
          }
          if (!load_v(j)) break;
          nv = j + 1;
          USP_TRACE_EV(1, j);
        }
      }
      if (*abort_flag) {
        // Let the copies this thread started land before the CTA exits.
        for (int j = (nk > C::KSTAGES ? nk - C::KSTAGES : 0); j < nk; ++j)
          mbar_wait_drain(&bars->k_full[j % C::KSTAGES], (j / C::KSTAGES) & 1, kDrainLimitNs);
        for (int j = (nv > C::VSTAGES ? nv - C::VSTAGES : 0); j < nv; ++j)
          mbar_wait_drain(&bars->v_full[j % C::VSTAGES], (j / C::VSTAGES) & 1, kDrainLimitNs);
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
      auto issue_pv = [&](int i) -> bool {
        const int st = i % C::VSTAGES;
        if (!mbar_wait(&bars->v_full[st], (i / C::VSTAGES) & 1, abort_flag, &g_attn_error, 21, kWaitLimitNs)) return false;
        if (!mbar_wait(&bars->p_full[i & 1], (i >> 1) & 1, abort_flag, &g_attn_error, 22, kWaitLimitNs)) return false;
        USP_TRACE_EV(3, i);
        tc_fence_after();
        const uint32_t pcol = tmem + ((i & 1) ? kColP1 : kColP0);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = make_smem_desc(v_addr + st * C::TILE_BYTES + kk * 16 * C::ROWB, C::BLOCK_BYTES,
                                                C::SBO, C::LAYOUT);
          umma_ts(tmem + kColO, pcol + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->pv_done[i & 1]);
        USP_TRACE_EV(4, i);
        umma_commit(&bars->v_empty[st]);
        return true;
      };
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % C::KSTAGES;
        if (!mbar_wait(&bars->k_full[st], (j / C::KSTAGES) & 1, abort_flag, &g_attn_error, 23, kWaitLimitNs)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&bars->s_empty[j & 1], ((j - 2) >> 1) & 1, abort_flag, &g_attn_error, 24, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t scol = tmem + ((j & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int e = kk * 16;
          const uint32_t off = (e / C::ATOM) * C::BLOCK_BYTES + (e % C::ATOM) * 2;
          const uint64_t adesc = make_smem_desc(q_addr + off, 16, C::SBO, C::LAYOUT);
          const uint64_t bdesc = make_smem_desc(k_addr + st * C::TILE_BYTES + off, 16, C::SBO, C::LAYOUT);
          umma_ss(scol, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[j & 1]);
        USP_TRACE_EV(2, j);
        umma_commit(&bars->k_empty[st]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(ntiles - 1);
      if (ok) umma_commit(&bars->o_full);
      // All MMAs this thread issued must finish before TMEM is released.
      umma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    // Warps w and w+4 share TMEM lane quarter w%4 (32 query rows, one per
    // thread); warp w takes key columns [0, 64) of each tile and warp w+4
    // columns [64, 128). The two swap partial row maxima through shared
    // memory (exchange barrier per pair), keep separate partial row sums, and
    // split the O columns for the rescale and the epilogue.
    const int quarter = warp & 3;
    const int half = warp >> 2;                      // 0 or 1
    const int row = quarter * 32 + lane;             // TMEM lane = query row in the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    constexpr int kHalf = kBN / 2;                   // key columns per thread
    constexpr int kOChunks = D / 16;
    constexpr int kOChunks0 = (kOChunks + 1) / 2;    // O chunks of half 0
    const int oc_lo = half ? kOChunks0 : 0;
    const int oc_hi = half ? kOChunks : kOChunks0;
    float* xch = bars->xch;                          // [2 parity][2 half][128 rows]
    uint64_t* xbar = &bars->xbar[quarter];
    const float sl2 = p.scale_log2;
    float m = -INFINITY;  // running maximum, log2 domain (identical in both halves)
    float l = 0.f;        // this half's running denominator
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, &g_attn_error, 30, kWaitLimitNs))) { ok = false; break; }
      if (threadIdx.x == 0) USP_TRACE_EV(5, j);
      tc_fence_after();
      uint32_t sr[kHalf];
      const uint32_t scol = lane_addr + ((j & 1) ? kColS1 : kColS0) + half * kHalf;
      tmem_ld32(scol, sr);
      tmem_ld32(scol + 32, sr + 32);
      tmem_wait_ld();
      if (threadIdx.x == 0) USP_TRACE_EV(6, j);
      tc_fence_before();
      mbar_arrive(&bars->s_empty[j & 1]);

      float* s = reinterpret_cast<float*>(sr);
      const int valid = T - j * kBN - half * kHalf;  // valid columns of this half
      if (valid < kHalf) {
#pragma unroll
        for (int c = 0; c < kHalf; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      // Partial row maximum: four independent three-input chains, then a tree.
      float mx4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a = fmaxf(s[i], s[i + 4]);
#pragma unroll
        for (int c = i + 8; c < kHalf; c += 8) a = max3(a, s[c], s[c + 4]);
        mx4[i] = a;
      }
      const float pm = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      // Swap partial maxima with the partner warp.
      xch[((j & 1) * 2 + half) * kBM + row] = pm;
      mbar_arrive(xbar);
      if (!__all_sync(0xffffffffu, mbar_wait(xbar, j & 1, abort_flag, &g_attn_error, 34, kWaitLimitNs))) { ok = false; break; }
      const float mx = fmaxf(pm, xch[((j & 1) * 2 + (half ^ 1)) * kBM + row]);
      if (threadIdx.x == 0) USP_TRACE_EV(7, j);
      const float m_new = fmaxf(m, mx * sl2);
      if (j == 0) {
        m = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m + kRescaleThreshold)) {
        // O holds sum_{i<j} exp2(s_i - m) v_i; bring it to the new maximum.
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, &g_attn_error, 31, kWaitLimitNs))) { ok = false; break; }
        tc_fence_after();
        const float alpha = ex2_approx(m - m_new);
        m = m_new;
        l *= alpha;
        for (int c = oc_lo; c < oc_hi; ++c) {
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
      // On full halves one pair in kPolyEvery takes the FMA-pipe exp2 so that
      // the MUFU pipe is not the only exp unit; masked halves use MUFU only, so
      // masked entries are exactly 0.
      uint32_t pk[kHalf / 2];
      uint64_t acc[4] = {0, 0, 0, 0};
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m, -m);
      if (valid >= kHalf) {
#pragma unroll
        for (int c = 0; c < kHalf; c += 2) {
          const uint64_t x = f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, negm2);
          float x0, x1;
          f2_unpack(x, x0, x1);
          uint64_t pp;
          if ((c / 2) % kPolyEvery == kPolyEvery - 1)
            pp = exp2_poly_f2(f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f)));
          else
            pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
          acc[(c / 2) & 3] = f2_add(acc[(c / 2) & 3], pp);
          float p0, p1;
          f2_unpack(pp, p0, p1);
          pk[c / 2] = pack2(p0, p1, BF16);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kHalf; c += 2) {
          const uint64_t x = f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, negm2);
          float x0, x1;
          f2_unpack(x, x0, x1);
          const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
          acc[(c / 2) & 3] = f2_add(acc[(c / 2) & 3], pp);
          float p0, p1;
          f2_unpack(pp, p0, p1);
          pk[c / 2] = pack2(p0, p1, BF16);
        }
      }
      {
        const uint64_t a01 = f2_add(acc[0], acc[1]);
        const uint64_t a23 = f2_add(acc[2], acc[3]);
        float u0, u1;
        f2_unpack(f2_add(a01, a23), u0, u1);
        l += u0 + u1;
      }
      // P buffer j%2 was last read by P_{j-2} V_{j-2}.
      if (threadIdx.x == 0) USP_TRACE_EV(8, j);
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[j & 1], ((j - 2) >> 1) & 1, abort_flag, &g_attn_error, 32, kWaitLimitNs))) { ok = false; break; }
      tc_fence_after();
      tmem_st32(lane_addr + ((j & 1) ? kColP1 : kColP0) + half * (kHalf / 2), pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[j & 1]);
      if (threadIdx.x == 0) USP_TRACE_EV(9, j);
    }
    // Combine the two halves' denominators.
    if (ok) {
      xch[((ntiles & 1) * 2 + half) * kBM + row] = l;
      mbar_arrive(xbar);
      ok = __all_sync(0xffffffffu, mbar_wait(xbar, ntiles & 1, abort_flag, &g_attn_error, 35, kWaitLimitNs));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort_flag, &g_attn_error, 33, kWaitLimitNs))) {
      tc_fence_after();
      const float inv_l = 1.f / (l + xch[((ntiles & 1) * 2 + (half ^ 1)) * kBM + row]);
      const int t = qtile * kBM + row;
      const AttnOut& out = p.out;
      // Destination(s) of this row.
      int seg_lo = 0, seg_hi = 0;
      int64_t row_in_seg = 0;
      if (t < T) {
        if (t < out.prefix) {
          seg_lo = 0;
          seg_hi = out.nseg;
          row_in_seg = t;
        } else {
          const int64_t tok = t - out.prefix;
          int s = 0;
          while (s + 1 < out.nseg && tok >= out.seg_start[s + 1]) ++s;
          seg_lo = s;
          seg_hi = s + 1;
          row_in_seg = out.prefix + tok - out.seg_start[s];
        }
      }
      for (int c = oc_lo; c < oc_hi; ++c) {
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
          const int64_t elem = ((static_cast<int64_t>(b) * rows_s + row_in_seg) * out.out_heads + hm) * D + c * 16;
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

// -------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

int make_map(CUtensorMap* map, const void* base, const AttnLaunch& L, int atom) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int e = 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(L.head_dim), static_cast<cuuint64_t>(L.in.head_extent),
                        static_cast<cuuint64_t>(L.tokens), static_cast<cuuint64_t>(L.batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(L.in.stride_head * e), static_cast<cuuint64_t>(L.in.stride_token * e),
                           static_cast<cuuint64_t>(L.in.stride_batch * e)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(atom), 1, kBM, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMapSwizzle swz = atom == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                      : (atom == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  CUtensorMapDataType dt = L.dtype == USP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(USP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return USP_OK;
}

template <int D, bool BF16>
int launch_d(const AttnLaunch& L, cudaStream_t stream) {
  using C = Cfg<D>;
  static_assert(C::SMEM_BYTES <= 232448, "shared memory above the 227 KB per-CTA limit");
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute(attention smem)");
    configured = true;
  }
  TcParams p;
  memset(&p, 0, sizeof(p));
  int rc;
  if ((rc = make_map(&p.tm_q, L.in.q, L, C::ATOM)) != USP_OK) return rc;
  if ((rc = make_map(&p.tm_k, L.in.k, L, C::ATOM)) != USP_OK) return rc;
  if ((rc = make_map(&p.tm_v, L.in.v, L, C::ATOM)) != USP_OK) return rc;
  p.out = L.out;
  p.tokens = L.tokens;
  p.batch = L.batch;
  p.n_heads = L.n_heads;
  p.scale_log2 = static_cast<float>(static_cast<double>(L.scale) * 1.4426950408889634);
  for (int i = 0; i < L.n_heads; ++i) p.heads[i] = L.heads[i];
  dim3 grid((L.tokens + kBM - 1) / kBM, L.batch * L.n_heads);
  attn_tc_kernel<D, BF16><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
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
  return L.dtype == USP_BF16 ? launch_dtype<true>(L, stream) : launch_dtype<false>(L, stream);
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
