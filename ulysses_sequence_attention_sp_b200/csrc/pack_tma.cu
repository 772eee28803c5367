// TMA-staged seq->head pack ("h3_blackwell_runtime/distributed.py -- Ragged
// Ulysses sequence-parallel transport", SequenceParallelContext.seq_to_heads),
// and the same move backwards (heads_to_seq): the permutation of
// permute_kernel, moved by the Tensor Memory Accelerator instead of vector
// loads and stores. Backwards, each unit's box is loaded from the head shard
// and stored to the sequence shard; the replicated prefix rows land in rank
// 0's shard only (the caller copies them to the others).
//
// A work unit is one head unit (D elements) of n consecutive token rows of one
// source rank: a 4-D tile load (d, head, row, batch) of box (D, 1, n, 1) from
// the source's sequence shard into shared memory, then a tile store of the
// same box into the destination head shard at the rows' token offset. Both
// tensor maps name the head and token axes with their real strides, so the
// transposition from [row][head] to [head][token] costs nothing. A tile holds
// hb consecutive head units (hb divides every buffer's selected head count).
// One thread per CTA issues the copies (loads complete on mbarriers, stores
// are tracked as bulk groups); the grid has one CTA per unit, each sized for
// a sixth of the shared memory, so many independent issuers run per SM. A
// CTA given several units (beyond the largest grid) pipelines them over
// kStages tiles. A source rank's last chunk is shifted back to
// end on the rank's last row, so no store ever reaches another rank's rows
// (the overlapped rows are written twice with the same bytes).
// No multicast: every load reads this device's own memory into its own CTA.
#include "device_common.cuh"
#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_pack_error;   // first wait that ran out (site code), 0 if none
__device__ uint32_t g_pack_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

namespace {

// Tiles sized for six CTAs per SM and one CTA per unit: measured on the
// reshard workload, 6.8 TB/s, against 6.05 for four persistent CTAs per SM
// looping over units with three tiles in flight each, and 5.75 for one CTA
// per unit with tiles sized for four CTAs (independent issuing threads
// matter more than tiles per thread).
constexpr int kCtasPerSm = 6;
constexpr int kStages = 2;
static_assert(kStages >= 2, "the pipeline loads one unit ahead of the store it waits for");
constexpr int kMaxRows = 64;                      // rows per unit (box height)
constexpr int64_t kSmemBudget = 200 * 1024 / kCtasPerSm;  // shared memory for one CTA's kStages tiles
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: only a broken copy waits this long
constexpr uint64_t kDrainLimitNs = 200000000ull;

struct PackTmaParams {
  CUtensorMap src[3][USP_MAX_WORLD];     // sequence-side buffers
  CUtensorMap dst[3][USP_MAX_WORLD];     // head-side buffers
  int64_t total_units;
  int32_t ntensors, n_seq, nsel, outer;
  int32_t dir;                           // 0: sequence -> head; 1: head -> sequence (same units, boxes swapped)
  int32_t hb;                            // head units per tile (divides every buffer's selected count)
  int32_t ngroups;                       // nsel / hb
  int32_t rows;                          // n
  uint32_t box_bytes;                    // bytes one tile copy moves
  uint32_t stage_bytes;                  // box_bytes rounded up to 128: TMA tile copies need 128-byte aligned smem
  int32_t r0[USP_MAX_WORLD];             // first source row of source s
  int32_t cnt[USP_MAX_WORLD];            // its row count
  int32_t d0[USP_MAX_WORLD];             // token offset of its first row on the head side
  int32_t chunk_prefix[USP_MAX_WORLD + 1];
  int32_t heads;                         // head units per sequence row (bounds-checking builds)
  int32_t buf_heads[USP_MAX_WORLD];      // head units of each head-side buffer
  int32_t full_tokens;                   // token rows of each head-side buffer
  uint16_t sel_head[USP_MAX_HEADS];      // head unit in the sequence row
  uint16_t sel_local[USP_MAX_HEADS];     // its index inside the owning head-side buffer
  uint8_t sel_rank[USP_MAX_HEADS];       // the owning head-side buffer
};

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int32_t c0, int32_t c1,
                                             int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group_0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct Unit {
  int t, b, s, i, row, tok;
};

__device__ __forceinline__ Unit unit_of(const PackTmaParams& p, int64_t u) {
  // u = ((t * outer + b) * chunks + k) * ngroups + g: head groups fastest, so
  // consecutive units read the same source rows. r.i is the group's first
  // selected head.
  Unit r;
  const int64_t chunks = p.chunk_prefix[p.n_seq];
  r.i = static_cast<int>(u % p.ngroups) * p.hb;
  int64_t q = u / p.ngroups;
  const int k = static_cast<int>(q % chunks);
  q /= chunks;
  r.b = static_cast<int>(q % p.outer);
  r.t = static_cast<int>(q / p.outer);
  int s = 0;
  while (s + 1 < p.n_seq && k >= p.chunk_prefix[s + 1]) ++s;
  r.s = s;
  int off = (k - p.chunk_prefix[s]) * p.rows;
  if (off > p.cnt[s] - p.rows) off = p.cnt[s] - p.rows;  // the last chunk ends on the rank's last row
  r.row = p.r0[s] + off;
  r.tok = p.d0[s] + off;
  return r;
}

__global__ void __launch_bounds__(32, 1) pack_tma_kernel(const __grid_constant__ PackTmaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full[kStages];
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;  // one issuing thread; the others have nothing to do
  for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
  abort_flag = (*reinterpret_cast<volatile uint32_t*>(&g_pack_error) != 0) ? 1 : 0;
  fence_mbar_init();
  if (abort_flag) return;

  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t mine = p.total_units > first ? (p.total_units - first + step - 1) / step : 0;
  auto load = [&](int64_t k) {
    const Unit u = unit_of(p, first + k * step);
    const int st = static_cast<int>(k % kStages);
    // bounds-checking builds: the tile stays inside the source rank's rows and heads
    // (the copy still runs, so the mbarrier completes; the site is recorded)
    in_bounds(u.row, p.rows, p.r0[u.s] + p.cnt[u.s], 61, &g_pack_bounds);
    in_bounds(p.sel_head[u.i], p.hb, p.heads, 62, &g_pack_bounds);
    mbar_arrive_expect_tx(&full[st], p.box_bytes);
    uint8_t* stage = smem + static_cast<size_t>(st) * p.stage_bytes;
    if (p.dir == 0)
      tma_load_4d(&p.src[u.t][u.s], &full[st], stage, 0, p.sel_head[u.i], u.row, u.b);
    else
      tma_load_4d(&p.dst[u.t][p.sel_rank[u.i]], &full[st], stage, 0, p.sel_local[u.i], u.tok, u.b);
  };
  const int64_t pro = mine < kStages - 1 ? mine : kStages - 1;
  for (int64_t k = 0; k < pro; ++k) load(k);
  int64_t issued = pro, k = 0;
  for (; k < mine; ++k) {
    const int st = static_cast<int>(k % kStages);
    if (!mbar_wait(&full[st], static_cast<uint32_t>((k / kStages) & 1), &abort_flag, &g_pack_error, 60,
                   kWaitLimitNs))
      break;
    fence_proxy_async_smem();  // the landed tile, seen by this thread, before the store reads it
    const Unit u = unit_of(p, first + k * step);
    if (!in_bounds(u.tok, p.rows, p.d0[u.s] + p.cnt[u.s], 63, &g_pack_bounds) ||
        !in_bounds(p.sel_local[u.i], p.hb, p.buf_heads[p.sel_rank[u.i]], 64, &g_pack_bounds) ||
        !in_bounds(u.tok, p.rows, p.full_tokens, 65, &g_pack_bounds)) {
      bulk_commit_group();  // an empty group keeps the stage accounting of wait_group.read
    } else {
      uint8_t* stage = smem + static_cast<size_t>(st) * p.stage_bytes;
      if (p.dir == 0)
        tma_store_4d(&p.dst[u.t][p.sel_rank[u.i]], stage, 0, p.sel_local[u.i], u.tok, u.b);
      else
        tma_store_4d(&p.src[u.t][u.s], stage, 0, p.sel_head[u.i], u.row, u.b);
      bulk_commit_group();
    }
    if (issued < mine) {
      bulk_wait_group_read_1();  // the store of unit k-1 has read its stage, which the next load reuses
      load(issued);
      ++issued;
    }
  }
  if (k < mine) {
    // A wait ran out: let the loads still in flight land before the CTA exits.
    for (int64_t j = k; j < issued; ++j)
      mbar_wait_drain(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1), kDrainLimitNs);
  }
  bulk_wait_group_0();  // every store has completed before the CTA exits
}

int encode(CUtensorMap* map, const void* base, int elem, int64_t dv, int64_t heads, int64_t rows, int64_t outer,
           int64_t head_stride, int64_t row_stride, int64_t outer_stride, int box_heads, int box_rows) {
  const uint64_t dims[4] = {static_cast<uint64_t>(dv), static_cast<uint64_t>(heads), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(outer)};
  const uint64_t strides[3] = {static_cast<uint64_t>(head_stride), static_cast<uint64_t>(row_stride),
                               static_cast<uint64_t>(outer_stride)};
  const uint32_t box[4] = {static_cast<uint32_t>(dv), static_cast<uint32_t>(box_heads),
                           static_cast<uint32_t>(box_rows), 1};
  const CUtensorMapDataType dt = elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  return encode_tiled_4d(map, dt, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace

bool pack_tma_supported(int elem, int64_t unit_bytes) {
  return (elem == 2 || elem == 4) && unit_bytes % 16 == 0 && unit_bytes / elem <= 256;
}

int launch_pack_tma(const PermuteArgs& a, int elem, int64_t unit_bytes, cudaStream_t stream) {
  if (a.dir != 0 && a.dir != 1) return set_error(USP_ERR_INVALID_ARG, "internal: bad direction %d", a.dir);
  if (a.nsel == 0 || a.seq_rows[a.n_seq] == 0) return USP_OK;
  const int64_t dv = unit_bytes / elem;
  if (!pack_tma_supported(elem, unit_bytes))
    return set_error(USP_ERR_UNSUPPORTED, "TMA pack needs head_dim * element size a multiple of 16 B and <= 256 elements");
  thread_local PackTmaParams p;  // ~25 KB: built on the host, copied into the launch's parameters
  memset(&p, 0, sizeof(p));
  p.ntensors = a.ntensors;
  p.dir = a.dir;
  p.n_seq = a.n_seq;
  p.nsel = a.nsel;
  p.outer = static_cast<int32_t>(a.outer);
  int32_t min_cnt = INT32_MAX;
  if (a.prefix > 0 && a.tok_start[0] != 0)
    return set_error(USP_ERR_INVALID_ARG, "internal: TMA pack with prefix rows needs source 0's tokens to start at 0");
  for (int s = 0; s < a.n_seq; ++s) {
    // Source 0's prefix rows and token rows form one run from head-side row 0
    // (its tokens start at token 0); other sources skip their prefix rows.
    const bool whole = s == 0 && a.prefix > 0;
    p.r0[s] = whole ? 0 : a.prefix;
    p.cnt[s] = static_cast<int32_t>(whole ? a.prefix + a.tok_len[s] : a.tok_len[s]);
    p.d0[s] = static_cast<int32_t>(whole ? 0 : a.prefix + a.tok_start[s]);
    if (p.cnt[s] < min_cnt) min_cnt = p.cnt[s];
  }
  // Head units per tile: the largest common divisor of the buffers' selected
  // head counts (the selected heads of a buffer are consecutive), so a tile
  // never spans two buffers. Box height: at most kMaxRows, the smallest
  // source's row count (so a shifted last chunk stays inside its source), and
  // kStages tiles within kSmemBudget bytes of shared memory.
  {
    int32_t count[USP_MAX_WORLD] = {};
    for (int i = 0; i < a.nsel; ++i) ++count[a.sel_rank[i]];
    int32_t g = 0;
    for (int r = 0; r < a.n_head; ++r) {
      int32_t x = count[r], y = g;
      while (y) { const int32_t t = x % y; x = y; y = t; }
      g = count[r] ? x : g;
    }
    // the largest divisor of g whose tile rows still leave room for 2+ rows per stage
    p.hb = 1;
    for (int32_t d = g; d > 1; --d)
      if (g % d == 0 && static_cast<int64_t>(d) * unit_bytes * kStages * 2 <= kSmemBudget) {
        p.hb = d;
        break;
      }
  }
  const int64_t tile_row = static_cast<int64_t>(p.hb) * unit_bytes;
  int64_t rows = (kSmemBudget / kStages - 127) / tile_row;  // a stage also rounds up to 128 bytes
  if (rows > kMaxRows) rows = kMaxRows;
  if (rows > min_cnt) rows = min_cnt;
  if (rows < 1) return set_error(USP_ERR_UNSUPPORTED, "TMA pack: a head unit of %lld bytes is too large",
                                 static_cast<long long>(unit_bytes));
  p.rows = static_cast<int32_t>(rows);
  p.ngroups = a.nsel / p.hb;
  p.box_bytes = static_cast<uint32_t>(p.rows * tile_row);
  p.stage_bytes = (p.box_bytes + 127u) & ~127u;
  p.chunk_prefix[0] = 0;
  for (int s = 0; s < a.n_seq; ++s) p.chunk_prefix[s + 1] = p.chunk_prefix[s] + (p.cnt[s] + p.rows - 1) / p.rows;
  for (int i = 0; i < a.nsel; ++i) {
    p.sel_head[i] = static_cast<uint16_t>(a.sel_head[i] - a.seq_unit_base);
    p.sel_rank[i] = a.sel_rank[i];
    p.sel_local[i] = static_cast<uint16_t>(a.sel_head[i] - a.head_start[a.sel_rank[i]]);
  }
  p.total_units = static_cast<int64_t>(a.ntensors) * a.outer * p.chunk_prefix[a.n_seq] * p.ngroups;
  p.heads = a.heads;
  p.full_tokens = static_cast<int32_t>(a.full_tokens);
  for (int r = 0; r < a.n_head; ++r) p.buf_heads[r] = head_units(a, r);
  int rc;
  for (int t = 0; t < a.ntensors; ++t) {
    for (int s = 0; s < a.n_seq; ++s) {
      const int64_t rows_s = a.prefix + a.tok_len[s];
      if ((rc = encode(&p.src[t][s], a.seq_ptr[t][s], elem, dv, a.heads, rows_s, a.outer, unit_bytes,
                       a.heads * unit_bytes, rows_s * a.heads * unit_bytes, p.hb, p.rows)) != USP_OK)
        return rc;
    }
    for (int r = 0; r < a.n_head; ++r) {
      const int64_t c = head_units(a, r);
      if (c == 0) continue;
      const int64_t ft = a.full_tokens;
      const bool head_major = a.head_layout == 1;  // [C][outer][full][unit], else [outer][full][C][unit]
      if ((rc = encode(&p.dst[t][r], a.head_ptr[t][r], elem, dv, c, ft, a.outer,
                       head_major ? a.outer * ft * unit_bytes : unit_bytes,
                       head_major ? unit_bytes : c * unit_bytes,
                       head_major ? ft * unit_bytes : ft * c * unit_bytes, p.hb, p.rows)) != USP_OK)
        return rc;
    }
  }
  const size_t smem = static_cast<size_t>(kStages) * p.stage_bytes + 128;  // + alignment of the base
  if (int rc = ensure_smem_limit(reinterpret_cast<const void*>(pack_tma_kernel), smem, "cudaFuncSetAttribute(pack smem)"))
    return rc;
  const unsigned grid = static_cast<unsigned>(p.total_units < 0x7fffffff ? p.total_units : 0x7fffffff);
  pack_tma_kernel<<<grid, 32, smem, stream>>>(p);
  count_launch();
  return cuda_check(cudaGetLastError(), "TMA pack launch");
}

int read_pack_bounds(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_pack_bounds, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read pack bounds word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_pack_bounds, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset pack bounds word");
  }
  return USP_OK;
}

int read_pack_error(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_pack_error, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read pack error word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_pack_error, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset pack error word");
  }
  return USP_OK;
}

}  // namespace usp
