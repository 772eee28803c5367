// Host-side internals shared by the C ABI (plan.cpp) and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "usp.h"

struct usp_plan {
  int64_t batch = 0;
  int64_t seq_len = 0;  // T, tokens split across ranks
  int32_t heads = 0;
  int32_t head_dim = 0;
  int32_t world = 0;
  int32_t dtype = 0;
  int32_t prefix = 0;   // replicated leading tokens
  int32_t elem = 0;     // bytes per element
  int64_t tok_start[USP_MAX_WORLD] = {};
  int64_t tok_len[USP_MAX_WORLD] = {};
  int32_t head_start[USP_MAX_WORLD + 1] = {};
  int32_t head_len[USP_MAX_WORLD] = {};
  int32_t group_heads = 0;  // largest per-rank head count (rank 0's)
  int32_t heads_kv = 0;     // k/v heads (== heads without grouped-query attention)
  int32_t kv_group = 1;     // query heads per kv head
  int32_t kv_head_start[USP_MAX_WORLD + 1] = {};
  int32_t kv_head_len[USP_MAX_WORLD] = {};
  // Ulysses + Ring hybrid: heads are split over `head_ranks` = ulysses ranks
  // (the head arrays above hold head_ranks entries); `ring` Ulysses groups of
  // consecutive ranks. The plain block is head_ranks == world, ring == 1.
  int32_t head_ranks = 0;
  int32_t ring = 1;
  int32_t pack_mode = USP_PACK_TMA;  // USP_PACK_TMA (default) or USP_PACK_VECTOR: how seq->head packs move data
  int32_t attn_ctas = 0;  // cap on the attention kernel's CTAs (0: automatic)
  int32_t attn_kernel = USP_ATTN_AUTO;  // which tensor-core attention kernel (usp_plan_set_attention_kernel)
  int device = 0;
  cudaStream_t aux = nullptr;             // runs the per-chunk seq->head packs
  cudaEvent_t ev_inputs = nullptr;        // caller stream -> aux: inputs ready
  std::vector<cudaEvent_t> ev_chunk;      // aux -> caller stream: chunk c packed
  cudaEvent_t t_start = nullptr;          // caller-owned timing events (profiling hook)
  cudaEvent_t t_stop = nullptr;
  // Held while one call enqueues its work (event records, waits and launches
  // on the caller's stream and on `aux`), so that calls from several host
  // threads never interleave their event records and waits. Recursive: the
  // graph capture holds it around the call it captures.
  mutable std::recursive_mutex lock;
  // Device address of the allocation-free entry point's fixed scratch array on
  // this plan's device, looked up when the plan is created (the plan lives no
  // longer than the CUDA context it was created in).
  void* noalloc_scratch = nullptr;

  int64_t tokens() const { return prefix + seq_len; }
};

namespace usp {

int set_error(int code, const char* fmt, ...);
void count_launch();
int cuda_check(cudaError_t e, const char* what);

// ------------------------------------------------------------ permutation
// One kernel moves rows between "sequence-side" buffers (each holds whole
// token rows of H head units) and "head-side" buffers (each holds a
// contiguous range of head units for every token). All layout operations of
// the block are instances of it (see plan.cpp).
struct PermuteArgs {
  int32_t dir;          // 0: sequence side -> head side; 1: head side -> sequence side
  int32_t n_seq;        // sequence-side buffers
  int32_t n_head;       // head-side buffers
  int32_t ntensors;     // tensors moved per launch (same geometry), 1..3
  int32_t prefix;       // replicated leading rows of every sequence-side buffer
  int32_t heads;        // head units per sequence-side row
  int32_t dv;           // vectors per head unit
  int32_t head_layout;  // 0: [outer][full_tokens][C_r][dv]; 1: [C_r][outer][full_tokens][dv]
  int32_t nsel;         // head units moved (a head chunk selects a subset)
  int32_t unit_batches; // unrolled batches of a row per work unit (set by launch_permute)
  int64_t outer;        // batch
  int64_t full_tokens;  // rows per batch element on the head side (prefix + T)
  int64_t seq_rows[USP_MAX_WORLD + 1];  // prefix sums of outer * (prefix + T_s)
  int64_t tok_start[USP_MAX_WORLD];     // token offset of sequence buffer s (prefix excluded)
  int64_t tok_len[USP_MAX_WORLD];
  int32_t head_start[USP_MAX_WORLD + 1];  // head-unit range of head-side buffer r
  uint16_t sel_head[USP_MAX_HEADS];       // moved head units, ascending
  uint8_t sel_rank[USP_MAX_HEADS];        // head-side buffer owning each moved unit
  // Optional: explicit unit counts of the head-side buffers (explicit_counts
  // != 0), for buffers whose unit ranges leave gaps (one head chunk of every
  // rank); otherwise buffer r holds units [head_start[r], head_start[r+1]).
  int32_t explicit_counts;
  // Sequence-side rows hold units [seq_unit_base, seq_unit_base + heads) of the
  // head numbering (a row of one head chunk); 0 for whole rows.
  int32_t seq_unit_base;
  int32_t head_count[USP_MAX_WORLD];
  void* seq_ptr[3][USP_MAX_WORLD];
  void* head_ptr[3][USP_MAX_WORLD];
  int64_t seq_ext[USP_MAX_WORLD];   // vectors in sequence-side buffer s (set by launch_permute)
  int64_t head_ext[USP_MAX_WORLD];  // vectors in head-side buffer r (set by launch_permute)
};

// vec_bytes in {16, 8, 4, 2}; dv counts vectors of that size.
// Units held by head-side buffer r.
__host__ __device__ inline int32_t head_units(const PermuteArgs& a, int r) {
  return a.explicit_counts ? a.head_count[r] : a.head_start[r + 1] - a.head_start[r];
}

int launch_permute(const PermuteArgs& a, int vec_bytes, cudaStream_t stream);

// Bounds-checking builds: the first out-of-range site each copy kernel
// recorded (0 if none), read and optionally reset, per translation unit.
int read_permute_bounds(uint32_t* code, bool reset);
int read_rows_bounds(uint32_t* code, bool reset);
int read_attention_bounds(uint32_t* code, bool reset);
int read_simt_bounds(uint32_t* code, bool reset);
int read_pack_bounds(uint32_t* code, bool reset);

// The same sequence -> head permutation (dir 0) moved by TMA tile copies
// (pack_tma.cu); unit_bytes = bytes of one head unit. Needs 2- or 4-byte
// elements and unit_bytes a multiple of 16 of at most 256 elements.
bool pack_tma_supported(int elem, int64_t unit_bytes);
int launch_pack_tma(const PermuteArgs& a, int elem, int64_t unit_bytes, cudaStream_t stream);
int read_pack_error(uint32_t* code, bool reset);

int sm_count();

// Raises kernel `func`'s dynamic shared-memory limit to at least `bytes` on the
// current device, and (carveout >= 0) sets its preferred shared-memory carveout
// in percent. The attributes are per device, so the value set is remembered
// per (kernel, device); thread-safe.
int ensure_smem_limit(const void* func, size_t bytes, const char* what, int carveout = -1);

// The plan's device-free part (sizes, splits, grouped-query check): plan.cpp.
int plan_geometry(usp_plan* p, int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv, int32_t head_dim,
                  int32_t ulysses_size, int32_t ring_size, int32_t dtype, int32_t prefix_tokens);

// Device address of the allocation-free entry point's scratch array on the
// current device (noalloc.cu).
int noalloc_scratch_lookup(void** out);

// ------------------------------------------------------- row collectives
// Ragged row collectives over the plan's token split. Rank r's local buffer is
// [outer][tok_len[r]][nv vectors]; a full buffer is [outer][total_rows][nv].
// all_gather_rows: src = local buffers, dst = full buffers (one per rank).
// reduce_scatter_rows: src = full partials, dst = local buffers.
struct RowsArgs {
  int32_t world;
  int32_t pad0;
  int64_t outer;
  int64_t total_rows;
  int64_t nv;  // vectors per row
  int64_t tok_start[USP_MAX_WORLD];
  int64_t tok_len[USP_MAX_WORLD];
  int64_t seg_tiles[USP_MAX_WORLD];        // set by the launcher
  int64_t tile_prefix[USP_MAX_WORLD + 1];  // set by the launcher
  const void* src[USP_MAX_WORLD];
  void* dst[USP_MAX_WORLD];
};

int launch_all_gather_rows(const RowsArgs& a, int vec_bytes, cudaStream_t stream);

// ------------------------------------------------- segmented row copy
// scatter_sequence / gather_sequence: every kind s of segment is a run of
// rows[s] rows that is contiguous, within each of the `outer` batch elements,
// in both buffers: rows [srow0[s], +rows[s]) of shard `shard[s]`, laid out
// [outer][shard_rows[s]][nv], and rows [frow0[s], +rows[s]) of the full buffer
// [outer][full_rows][nv]. nv counts 16-byte vectors per row.
constexpr int kMaxCopyKinds = 2 * USP_MAX_WORLD;  // every rank's token window + the prefix rows
struct CopyArgs {
  int32_t to_shards;  // 1: full -> shards (scatter), 0: shards -> full (gather)
  int32_t nkinds;
  int64_t outer;
  int64_t nv;
  int64_t full_rows;
  int32_t shard[kMaxCopyKinds];
  int64_t shard_rows[kMaxCopyKinds];
  int64_t srow0[kMaxCopyKinds];
  int64_t frow0[kMaxCopyKinds];
  int64_t rows[kMaxCopyKinds];
  int64_t seg_tiles[kMaxCopyKinds];        // set by the launcher
  int64_t tile_prefix[kMaxCopyKinds + 1];  // set by the launcher
  void* full;
  void* shards[USP_MAX_WORLD];
};

int launch_copy_rows(const CopyArgs& a, cudaStream_t stream);
int launch_reduce_scatter_rows(const RowsArgs& a, int vec_bytes, int dtype, cudaStream_t stream);

// -------------------------------------------------------------- attention
// Where output rows go. Row t of (batch b, head g): rows t < prefix go to every
// segment; other rows go to the segment s whose token range holds t - prefix.
// Address (elements): ptr_s + ((b * (prefix + len_s) + row_in_s) * out_heads + g - head_base) * D.
struct AttnOut {
  int32_t nseg;
  int32_t prefix;
  int32_t out_heads;
  int32_t head_base;  // head coordinate g is written at head g - head_base of a segment row
  int64_t seg_start[USP_MAX_WORLD];
  int64_t seg_len[USP_MAX_WORLD];
  void* seg_ptr[USP_MAX_WORLD];
};

// A 4-D view (d, head, token, batch) of one operand.
struct AttnView {
  int64_t stride_head;   // elements
  int64_t stride_token;  // elements
  int64_t stride_batch;  // elements
  int64_t head_extent;   // head coordinates in the view
};

// The launch processes every q head coordinate in heads[0..n_heads) for every
// batch element; q head coordinate h reads k/v head coordinate
// (q_head_base + h) / kv_group - kv_head_base (grouped-query attention).
struct AttnInputs {
  const void* q;
  const void* k;
  const void* v;
  AttnView qv;
  AttnView kvv;
  int32_t kv_group;
  int32_t q_head_base;
  int32_t kv_head_base;
  int32_t pad0;
};

// Query groups and key blocks of a launch (the Ulysses + Ring hybrid). Query
// group g is rows [q_start[g], q_start[g+1]) of the q view's token axis; key
// block k is rows [kv_start[k], kv_start[k+1]) of the k/v views' token axis.
// Group g takes the key blocks in ring order g, g-1, ..., g-n_kvblocks+1
// (mod n_kvblocks) and the online softmax carries its state across them.
// n_qgroups = 0 means one group [0, tokens); n_kvblocks = 0 one block
// [0, kv_tokens). Every group and block is non-empty.
struct AttnBlocks {
  int32_t n_qgroups;
  int32_t n_kvblocks;
  int32_t q_start[USP_MAX_WORLD + 1];
  int32_t kv_start[USP_MAX_WORLD + 1];
};

struct AttnLaunch {
  AttnInputs in;
  AttnOut out;
  AttnBlocks blocks;
  float* lse;         // optional: [q head coordinate][batch][tokens] fp32, log-sum-exp (natural log) of the scaled scores
  int32_t kv_tokens;  // rows of the k/v views (0: tokens)
  int32_t tokens;  // T' (queries per head; keys too unless kv_tokens is set)
  int32_t batch;
  int32_t n_heads;
  int32_t head_dim;
  int32_t dtype;
  float scale;
  int32_t max_ctas;  // cap on the tensor-core kernel's CTAs (0: automatic)
  int32_t kernel;    // USP_ATTN_AUTO, USP_ATTN_ONE_TILE or USP_ATTN_TWO_TILE
  uint16_t heads[USP_MAX_HEADS];
};

// Resolves the launch's AttnBlocks (defaults: one group, one block) into
// explicit tables, with q_tile_prefix[g] = query tiles of `rows_per_tile` rows
// before group g. Returns false if a table is not increasing from 0 <= start
// to an end within the token counts.
inline bool fill_blocks(const AttnLaunch& L, int kv_tokens, int rows_per_tile, int32_t& nq, int32_t& nk,
                        int32_t* q_start, int32_t* q_tile_prefix, int32_t* kv_start) {
  nq = L.blocks.n_qgroups > 0 ? L.blocks.n_qgroups : 1;
  nk = L.blocks.n_kvblocks > 0 ? L.blocks.n_kvblocks : 1;
  if (nq > USP_MAX_WORLD || nk > USP_MAX_WORLD) return false;
  for (int i = 0; i <= nq; ++i) q_start[i] = L.blocks.n_qgroups > 0 ? L.blocks.q_start[i] : (i ? L.tokens : 0);
  for (int i = 0; i <= nk; ++i) kv_start[i] = L.blocks.n_kvblocks > 0 ? L.blocks.kv_start[i] : (i ? kv_tokens : 0);
  if (q_start[0] < 0 || q_start[nq] > L.tokens || kv_start[0] < 0 || kv_start[nk] > kv_tokens) return false;
  q_tile_prefix[0] = 0;
  for (int g = 0; g < nq; ++g) {
    if (q_start[g + 1] <= q_start[g]) return false;
    q_tile_prefix[g + 1] = q_tile_prefix[g] + (q_start[g + 1] - q_start[g] + rows_per_tile - 1) / rows_per_tile;
  }
  for (int k = 0; k < nk; ++k)
    if (kv_start[k + 1] <= kv_start[k]) return false;
  return true;
}

// A 4-D tiled TMA map with no interleave, 256-byte L2 promotion and no
// out-of-bounds fill, through the driver's cuTensorMapEncodeTiled.
int encode_tiled_4d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4], CUtensorMapSwizzle swizzle);

// 4-D TMA map (d, head, token, batch) of one 16-bit attention operand view
// with `rows` tokens; boxes of `atom` elements x 1 head x box_rows tokens,
// swizzled by the atom width (64: 128 B, 32: 64 B, 16: 32 B).
int make_map(CUtensorMap* map, const void* base, const AttnView& view, const AttnLaunch& L, int64_t rows, int atom,
             int box_rows);

bool attention_tc_supported(int dtype, int head_dim);
// Two query tiles per CTA (attn_pp.cu): 16-bit, head_dim 64..128 in steps of 16.
bool attention_pp_supported(int dtype, int head_dim, int kernel = USP_ATTN_TWO_TILE);
int launch_attention_pp(const AttnLaunch& L, cudaStream_t stream);
int read_pp_error(uint32_t* code, bool reset);
int read_pp_bounds(uint32_t* code, bool reset);
int launch_attention_tc(const AttnLaunch& L, cudaStream_t stream);
int launch_attention_simt(const AttnLaunch& L, cudaStream_t stream);
int read_attention_error(uint32_t* code, bool reset);
int launch_wait_timeout_probe(uint32_t limit_us, cudaStream_t stream);

// Plan helpers shared by the entry points of plan.cpp and dist.cpp (plan.cpp).
int plan_vec_bytes(const usp_plan* plan);
int plan_launch_pack(const usp_plan* plan, const PermuteArgs& a, cudaStream_t stream);
int plan_check_ptr(const void* p, const char* what);
int plan_check_device(const usp_plan* plan);
int plan_check_attention(const usp_plan* plan);
int plan_launch_attention(const AttnLaunch& L, cudaStream_t stream);
float plan_scale(const usp_plan* plan, float scale);

}  // namespace usp
