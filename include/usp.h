/*
 * usp.h -- C ABI of libusp: the Ulysses sequence-parallel attention block on
 * one B200 (sm_100a), with P sequence-parallel ranks held as P virtual-rank
 * buffers in one device's memory.
 *
 * Conventions (every entry point):
 *  - Returns an int status, USP_OK (0) on success. On failure nothing has been
 *    launched, and usp_last_error_message() (thread-local) says why.
 *  - Device buffers are passed as plain device pointers and are owned by the
 *    caller; the library never frees them. The library owns only the plan
 *    (a host object plus one auxiliary CUDA stream and its events).
 *  - "Per-rank arrays" are host arrays of `world` device pointers, element r
 *    for virtual rank r; multi-tensor calls pass ntensors*world pointers,
 *    tensor-major (all ranks of tensor 0, then tensor 1, ...).
 *  - Every launch goes on the caller's stream (`stream`, a cudaStream_t; NULL
 *    is the legacy default stream). No call synchronises the host, except
 *    usp_device_status(). Calls are stream-ordered like any CUDA kernel.
 *  - Threads and streams: one plan may serve calls from several host threads
 *    and on several streams at once. Each call enqueues its work (including
 *    the event records and waits of usp_ulysses_attention's chunk overlap on
 *    the plan's auxiliary stream) under the plan's lock, so calls never
 *    cross-wire each other's dependencies; work of different calls is then
 *    ordered only by the streams it runs on. Calls that may run at the same
 *    time on the GPU must not share an output or a workspace buffer (the
 *    allocation-free entry point shares one scratch array: see there).
 *    Plan set-up calls (usp_plan_set_*) must not race with calls using the
 *    plan.
 *  - Tensors are dense and contiguous, row-major, in the BSHD layout of the
 *    ragged transport page: [batch, tokens, heads, head_dim]. Pointers must be
 *    16-byte aligned (USP_ERR_ALIGN otherwise); there is no slow path.
 *  - Element types: USP_BF16, USP_FP16 (2 bytes) and USP_FP32 (4 bytes).
 *    Layout operations copy bytes and are exact for any type.
 *
 * Notation: T = seq_len tokens split across ranks, prefix = replicated leading
 * tokens (a cls token; 0 or 1), T' = prefix + T, H = heads, D = head_dim,
 * B = batch, P = world. Rank r owns tokens [t0_r, t0_r + T_r) and heads
 * [h0_r, h0_r + H_r), both from the balanced split (earlier ranks take the
 * remainder). A sequence shard of rank r is [B, prefix + T_r, H, D]; a head
 * shard of rank r is [B, T', H_r, D].
 *
 * Sources: "mstar.model.components.distributed.sequence_parallel" (API page),
 * "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
 * transport", "maxdiffusion PR #428: experimental two-phase (head-chunked)
 * Ulysses all-to-all", "deepspeed/sequence/autosp_vit.py".
 */
#ifndef USP_H_
#define USP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define USP_MAX_WORLD 32   /* largest P */
#define USP_MAX_HEADS 256  /* largest H */

enum usp_status {
  USP_OK = 0,
  USP_ERR_INVALID_ARG = 1, /* null pointer, bad count, P < 1, T < P, H < P ...   */
  USP_ERR_SHAPE = 2,       /* sizes that do not fit the plan                      */
  USP_ERR_DTYPE = 3,       /* unknown element type                                */
  USP_ERR_ALIGN = 4,       /* pointer or row size not 16-byte aligned             */
  USP_ERR_CUDA = 5,        /* a CUDA runtime call failed (message has the name)    */
  USP_ERR_TIMEOUT = 6,     /* a device-side wait ran out (see usp_device_status)  */
  USP_ERR_UNSUPPORTED = 7, /* valid but not built (e.g. head_dim > 256)           */
  USP_ERR_NO_DEVICE = 8,   /* no CUDA device is visible                           */
  USP_ERR_BOUNDS = 9       /* a bounds-checking build (-DUSP_BOUNDS_CHECK) skipped an
                              out-of-range offset (see usp_device_status)          */
};

enum usp_dtype { USP_BF16 = 0, USP_FP32 = 1, USP_FP16 = 2 };

typedef struct usp_plan usp_plan;

/* Thread-local text of the last failure in this thread ("" if none). */
const char* usp_last_error_message(void);

/* Library version, major*10000 + minor*100 + patch. */
int usp_version(void);

/*
 * usp_balanced_ranges -- "h3_blackwell_runtime/distributed.py", balanced_ranges.
 * Splits `total` ordered items into `parts` contiguous non-empty ranges; the
 * first total % parts ranges are one longer. Writes parts starts and lengths.
 * USP_ERR_INVALID_ARG if parts < 1, total < parts, or an output is NULL.
 */
int usp_balanced_ranges(int64_t total, int32_t parts, int64_t* starts, int64_t* lengths);

/*
 * usp_seq_split -- API page, sp_seq_split: per-rank token counts summing to
 * `total`, earlier ranks taking the remainder. Writes `world` counts.
 * USP_ERR_INVALID_ARG if world < 1 or total < world (the transport page's rule).
 */
int usp_seq_split(int64_t total, int32_t world, int64_t* out_counts);

/*
 * usp_head_chunk_ranges -- "maxdiffusion PR #428", ulysses_attention_chunks:
 * local-head windows of the head-chunked passes. With s = ceil(G/num_chunks),
 * chunk c is [c*s, min((c+1)*s, G)); empty chunks are dropped. Writes the
 * number of chunks to *n_out and the windows to lo[]/hi[] (capacity >= G).
 * USP_ERR_INVALID_ARG if group_heads < 1 or num_chunks < 1.
 */
int usp_head_chunk_ranges(int32_t group_heads, int32_t num_chunks, int32_t* n_out, int32_t* lo,
                          int32_t* hi);

/*
 * usp_plan_create -- "h3_blackwell_runtime/distributed.py",
 * SequenceParallelContext.create: the token and head ownership of all P
 * virtual ranks (both balanced), for tensors of B x T' x H x D elements of
 * `dtype`, with `prefix_tokens` (0 or 1) replicated leading tokens
 * ("deepspeed/sequence/autosp_vit.py": the cls token is replicated on every
 * rank). Binds the plan to the current CUDA device and creates one auxiliary
 * stream and its events there (used to overlap head chunks), and looks up the
 * device address of usp_ulysses_attention_noalloc's scratch array there
 * (loading the library module that holds it reserves that array on the device,
 * once per process and device).
 * Errors: USP_ERR_INVALID_ARG (world < 1 or > USP_MAX_WORLD, seq_len < world,
 * heads < world or > USP_MAX_HEADS, batch < 1, head_dim < 1, prefix not 0/1),
 * USP_ERR_DTYPE, USP_ERR_NO_DEVICE, USP_ERR_CUDA.
 */
int usp_plan_create(usp_plan** out, int64_t batch, int64_t seq_len, int32_t heads,
                    int32_t head_dim, int32_t world, int32_t dtype, int32_t prefix_tokens);

/*
 * usp_plan_create_gqa -- as usp_plan_create, with grouped-query attention
 * (API page, ulysses_attention: q is [seq/P, Hq, D], k/v are [seq/P, Hkv, D]).
 * `heads` query heads and `heads_kv` k/v heads are each split by the balanced
 * rule; query head h uses kv head h / (heads / heads_kv). Errors as
 * usp_plan_create, plus USP_ERR_INVALID_ARG if heads is not a positive multiple
 * of heads_kv or heads_kv < world, and USP_ERR_SHAPE if some rank's query heads
 * use kv heads another rank owns (the API page's rule, both counts divisible by
 * world, always satisfies this). usp_plan_create is this call with
 * heads_kv = heads.
 */
int usp_plan_create_gqa(usp_plan** out, int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv,
                        int32_t head_dim, int32_t world, int32_t dtype, int32_t prefix_tokens);

/* Copies the plan's k/v head count and per-rank kv head ranges out; any output may be NULL. */
int usp_plan_query_kv(const usp_plan* plan, int32_t* heads_kv, int32_t* kv_head_start, int32_t* kv_head_len);

/*
 * usp_plan_create_hybrid -- the Ulysses + Ring hybrid ("maxdiffusion PR #428:
 * experimental two-phase (head-chunked) Ulysses all-to-all", which runs the
 * head-chunked passes on plain Ulysses and on Ulysses+Ring). world =
 * ulysses_size * ring_size virtual ranks split the tokens by the balanced
 * rule. Ulysses group g is ranks g*ulysses_size .. (g+1)*ulysses_size - 1 and
 * owns the contiguous token block of its members; inside a group the heads
 * (and kv heads) are split over the ulysses_size members by the balanced
 * rule, so rank r holds the heads of position u = r % ulysses_size. Ranks
 * with the same u form a ring that passes k/v blocks; outputs of the blocks
 * merge by their log-sum-exps. A prefix (cls) row is a key of block 0 only.
 * With such a plan, usp_ulysses_attention(_lse, _noalloc) run the hybrid
 * block, with the same arguments, workspace and chunking; scatter, gather and
 * the row collectives work as for any plan; the per-rank head-shard calls
 * (usp_ulysses_seq_to_head(_kv), usp_ulysses_head_to_seq, usp_sp_head_slice,
 * usp_sp_head_gather, usp_head_attention) return USP_ERR_UNSUPPORTED.
 * usp_plan_query reports rank r's head range as its position u's. Errors as
 * usp_plan_create_gqa, with USP_ERR_INVALID_ARG if ulysses_size * ring_size is
 * outside [1, USP_MAX_WORLD]. usp_plan_create_gqa is this call with
 * ring_size = 1 and ulysses_size = world.
 */
int usp_plan_create_hybrid(usp_plan** out, int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv,
                           int32_t head_dim, int32_t ulysses_size, int32_t ring_size, int32_t dtype,
                           int32_t prefix_tokens);

/*
 * usp_plan_set_pack_mode -- how this plan's sequence -> head moves
 * (usp_ulysses_seq_to_head(_kv) and the pack inside usp_ulysses_attention)
 * run. USP_PACK_TMA (the default): TMA tile copies, global -> shared ->
 * global, up to 64 rows of a few head units per tile, no multicast; used
 * where a head unit (head_dim * element size) is a multiple of 16 bytes of at
 * most 256 elements, the vector kernel otherwise. USP_PACK_VECTOR: 16-byte
 * vector loads and stores, one warp per segment of a sequence row. Both give identical bytes
 * ("h3_blackwell_runtime/distributed.py", seq_to_heads). Errors:
 * USP_ERR_INVALID_ARG for an unknown mode.
 */
#define USP_PACK_VECTOR 0
#define USP_PACK_TMA 1
int usp_plan_set_pack_mode(usp_plan* plan, int32_t mode);

/*
 * usp_plan_set_attention_ctas -- caps the CTAs of this plan's tensor-core
 * attention launches at max_ctas (0, the default: automatic). A launch with
 * more (query tile, batch, head) items than its CTAs runs persistent CTAs:
 * CTA c takes items c, c + max_ctas, ... and starts each item's loads and
 * first Q K^T under the previous item's last key tiles. Automatic mode uses
 * one CTA per SM when an item has at most 16 key tiles of 256 (short
 * sequences, where a CTA's fixed costs are a large share), and one CTA per
 * item otherwise. Under a cap (and with USP_ATTN_AUTO) the launch takes the
 * one-tile kernel; the USP_ATTN_TWO_CTA kernel, chosen explicitly, walks its
 * items with the cap's CTA count instead of two per SM; the
 * USP_ATTN_TWO_TILE kernel ignores the cap. A cap below the SM count leaves
 * SMs to kernels running beside the block on other streams. Results do not
 * depend on it (each item is computed the same way). The fp32 path ignores
 * it. Errors: USP_ERR_INVALID_ARG for max_ctas < 0.
 */
int usp_plan_set_attention_ctas(usp_plan* plan, int32_t max_ctas);

/*
 * usp_plan_set_attention_kernel -- which tensor-core attention kernel this
 * plan's 16-bit attention launches use (all compute the same function; see
 * usp_head_attention). USP_ATTN_ONE_TILE: one 128-row query tile per CTA with
 * 256-key tiles and four softmax threads per row (persistent CTAs for short
 * key sequences or under a CTA cap). USP_ATTN_TWO_TILE: two 128-row query
 * tiles per CTA with 128-key tiles and one softmax thread per row, the two
 * tiles' softmax and tensor-core work interleaved; head_dim a multiple of 16
 * in [64, 128]. USP_ATTN_TWO_CTA: the same kernel with one 128-row query tile
 * per CTA and two CTAs per SM, whose work the SM interleaves; head_dim 64 or
 * 80 (the two CTAs' K and V rings must fit in one SM's shared memory).
 * USP_ATTN_AUTO (the default), for launches without a CTA cap: TWO_TILE
 * where it applies and the launch has more than 16 key tiles of 256; with
 * fewer, TWO_CTA where it applies; ONE_TILE otherwise (and under a cap).
 * Results agree within rounding (the tile sizes differ, so the order of the
 * fp32 sums differs; TWO_TILE and TWO_CTA agree bit for bit). The fp32 path
 * ignores it. Errors:
 * USP_ERR_INVALID_ARG for an unknown value, USP_ERR_UNSUPPORTED for TWO_TILE
 * or TWO_CTA with another dtype or head_dim.
 */
#define USP_ATTN_AUTO 0
#define USP_ATTN_ONE_TILE 1
#define USP_ATTN_TWO_TILE 2
#define USP_ATTN_TWO_CTA 3
int usp_plan_set_attention_kernel(usp_plan* plan, int32_t kernel);

/* Copies the plan's Ulysses group size and ring size out (world and 1 for a plain plan); either may be NULL. */
int usp_plan_query_hybrid(const usp_plan* plan, int32_t* ulysses_size, int32_t* ring_size);

/* Releases the plan (synchronises its auxiliary stream first). NULL is ignored. */
int usp_plan_destroy(usp_plan* plan);

/* Copies the plan's ownership tables out; any output may be NULL. Arrays hold `world` entries. */
int usp_plan_query(const usp_plan* plan, int64_t* tok_start, int64_t* tok_len, int32_t* head_start,
                   int32_t* head_len);

/*
 * usp_scatter_sequence -- API page, scatter_sequence: each rank's contiguous
 * token window of a replicated tensor, materialised into that rank's buffer.
 * x_full is [outer, T', row] and x_shards[r] is [outer, prefix + T_r, row],
 * `row` = row_bytes bytes per token (a multiple of 16). The prefix rows are
 * copied to every shard. outer = 0 and row_bytes = 0 mean B and H*D*elem.
 */
int usp_scatter_sequence(const usp_plan* plan, const void* x_full, void* const* x_shards,
                         int64_t outer, int64_t row_bytes, void* stream);

/*
 * usp_gather_sequence -- API page, gather_sequence: the full tensor from the
 * shards in rank order (no padding is needed between virtual ranks). Shapes
 * as usp_scatter_sequence; the prefix rows are taken from rank 0.
 */
int usp_gather_sequence(const usp_plan* plan, const void* const* x_shards, void* x_full,
                        int64_t outer, int64_t row_bytes, void* stream);

/*
 * usp_sp_head_slice -- API page, sp_head_slice: rank r keeps heads
 * [h0_r, h0_r + H_r) of x_full [rows, H, D] into x_head_shards[r] [rows, H_r, D].
 * These are the heads the seq->head exchange routes to rank r. rows = 0 means B*T'.
 */
int usp_sp_head_slice(const usp_plan* plan, const void* x_full, void* const* x_head_shards,
                      int64_t rows, void* stream);

/* usp_sp_head_gather -- API page, sp_head_gather: inverse of usp_sp_head_slice. */
int usp_sp_head_gather(const usp_plan* plan, const void* const* x_head_shards, void* x_full,
                       int64_t rows, void* stream);

/*
 * usp_ulysses_seq_to_head -- "h3_blackwell_runtime/distributed.py",
 * SequenceParallelContext.seq_to_heads: for each of `ntensors` (1..3) tensors
 * (q, k, v), sequence shards in[t*P + i] [B, prefix+T_i, H, D] become head
 * shards out[t*P + r] [B, T', H_r, D]:
 *   out_r[b, prefix + t0_i + t, h, :] = in_i[b, prefix + t, h0_r + h, :]
 * and the prefix rows of every out_r come from rank 0's shard.
 * Outputs must not overlap inputs.
 */
int usp_ulysses_seq_to_head(const usp_plan* plan, int32_t ntensors, const void* const* in,
                            void* const* out, void* stream);

/*
 * usp_ulysses_seq_to_head_kv -- usp_ulysses_seq_to_head for k/v tensors under
 * grouped-query attention: sequence shards [B, prefix+T_i, Hkv, D] become head
 * shards [B, T', Hkv_r, D] over the plan's kv head ranges.
 */
int usp_ulysses_seq_to_head_kv(const usp_plan* plan, int32_t ntensors, const void* const* in, void* const* out,
                               void* stream);

/*
 * usp_ulysses_head_to_seq -- "h3_blackwell_runtime/distributed.py",
 * SequenceParallelContext.heads_to_seq: head shards in[t*P + r] [B, T', H_r, D]
 * become sequence shards out[t*P + i] [B, prefix+T_i, H, D]:
 *   out_i[b, prefix + t, h0_r + h, :] = in_r[b, prefix + t0_i + t, h, :]
 * and every rank receives the prefix rows.
 */
int usp_ulysses_head_to_seq(const usp_plan* plan, int32_t ntensors, const void* const* in,
                            void* const* out, void* stream);

/*
 * usp_all_gather_rows -- "h3_blackwell_runtime/distributed.py",
 * SequenceParallelContext.all_gather_rows: every rank receives all token rows,
 * concatenated in rank order, with no padding in the result.
 *   full_rows[r][b, t0_i + t, :] = local_rows[i][b, t, :]   for every r
 * local_rows[i] is [outer, T_i, row] and full_rows[r] is [outer, T, row] (T =
 * seq_len, the split tokens; the plan's prefix rows take no part), `row` =
 * row_bytes bytes, a multiple of 2. outer = 0 and row_bytes = 0 mean B and
 * H*D*elem. Caller-owned buffers, 16-byte aligned; outputs must not overlap
 * inputs or each other. One kernel launch; reads S and writes P*S bytes.
 * Errors: USP_ERR_INVALID_ARG (NULL pointer, bad sizes), USP_ERR_ALIGN,
 * USP_ERR_CUDA.
 */
int usp_all_gather_rows(const usp_plan* plan, const void* const* local_rows, void* const* full_rows,
                        int64_t outer, int64_t row_bytes, void* stream);

/*
 * usp_reduce_scatter_rows -- "h3_blackwell_runtime/distributed.py",
 * SequenceParallelContext.reduce_scatter_rows: every rank holds a partial sum
 * over all T token rows; rank r receives the sum over ranks of its own rows.
 *   local_rows[r][b, t, :] = sum_{i=0..P-1} partial_full_rows[i][b, t0_r + t, :]
 * partial_full_rows[i] is [outer, T, row] and local_rows[r] is [outer, T_r,
 * row] of the plan's dtype; row_bytes as usp_all_gather_rows (a multiple of
 * the element size). The sum runs in source-rank order in fp32 and is rounded
 * once (round to nearest even) to the storage type. Buffers as above. One
 * kernel launch; reads P*S and writes S bytes. Errors as usp_all_gather_rows.
 */
int usp_reduce_scatter_rows(const usp_plan* plan, const void* const* partial_full_rows, void* const* local_rows,
                            int64_t outer, int64_t row_bytes, void* stream);

/*
 * usp_head_attention -- API page, ulysses_attention's run_attention: the
 * unchanged single-device attention on every rank's head shard,
 *   o_r[b, :, h, :] = softmax(q_r[b, :, h, :] k_r[b, :, h, :]^T * scale) v_r[b, :, h, :]
 * non-causal, no mask, over all T' tokens ("deepspeed/sequence/autosp_vit.py":
 * ViT attention is non-causal). scale <= 0 selects 1/sqrt(D). 16-bit types
 * accumulate in fp32 on the tensor cores (tcgen05) with P rounded to the
 * input type; fp32 runs in fp32 on the CUDA cores. With grouped-query
 * attention k_r/v_r are [B, T', Hkv_r, D] and global query head h uses global
 * kv head h / (Hq / Hkv).
 */
int usp_head_attention(const usp_plan* plan, const void* const* q_heads, const void* const* k_heads,
                       const void* const* v_heads, void* const* o_heads, float scale, void* stream);

/*
 * usp_ulysses_attention_workspace_size -- bytes of device workspace that
 * usp_ulysses_attention needs (the head-sharded q, k and v of all ranks:
 * (Hq + 2 Hkv) * B * T' * D elements, each part 256-byte aligned).
 */
int usp_ulysses_attention_workspace_size(const usp_plan* plan, int32_t num_chunks, size_t* bytes);

/*
 * usp_ulysses_attention -- API page, ulysses_attention, with the head-chunked
 * passes of "maxdiffusion PR #428": sequence shards q/k/v[i]
 * [B, prefix+T_i, H, D] in (k/v with Hkv heads under grouped-query
 * attention), sequence shards out[i] [B, prefix+T_i, H, D] out.
 * For each head chunk c (usp_head_chunk_ranges over G = max H_r, the same
 * local-head window on every rank, clipped to H_r): the seq->head exchange of
 * chunk c's heads of q, k and v runs on the plan's auxiliary stream; the
 * attention of chunk c runs on `stream` once that exchange is done, and its
 * epilogue writes every output row straight to the sequence shard of the rank
 * that owns the row's token (the head->seq exchange, fused). The exchange of
 * chunk c+1 overlaps the attention of chunk c. The result does not depend on
 * num_chunks beyond rounding-free identity: heads are independent.
 * workspace: caller-owned device memory of at least
 * usp_ulysses_attention_workspace_size() bytes, 256-byte aligned; its
 * contents are scratch. Outputs must not overlap inputs or the workspace.
 */
int usp_ulysses_attention(const usp_plan* plan, const void* const* q, const void* const* k,
                          const void* const* v, void* const* out, float scale, int32_t num_chunks,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * usp_ulysses_attention_lse -- usp_ulysses_attention that also writes every
 * output row's log-sum-exp (the row statistic a ring step or a backward pass
 * merges with): lse[(h * B + b) * T' + t] = log sum_j exp(scale * q_t . k_j)
 * over all T' keys, natural log, fp32, h the global query head and t the row
 * in the full sequence (prefix rows first). lse is caller-owned device memory
 * of H * B * T' floats, 4-byte aligned. Errors as usp_ulysses_attention, plus
 * USP_ERR_INVALID_ARG for a NULL lse.
 */
int usp_ulysses_attention_lse(const usp_plan* plan, const void* const* q, const void* const* k,
                              const void* const* v, void* const* out, float* lse, float scale, int32_t num_chunks,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * usp_ulysses_attention_noalloc -- the source pages have no counterpart; this
 * entry point exists for callers that cannot allocate device memory when they
 * call the block, for example a plugin or custom operator whose host
 * framework owns all device memory and passes only the inputs and outputs, or
 * code on a path that must not synchronise the device (cudaFree does).
 *
 * It computes exactly what usp_ulysses_attention computes, with the same
 * arguments except the workspace: its scratch is a fixed array of
 * USP_NOALLOC_SCRATCH_BYTES inside the library's device memory, which every
 * GPU that loads the library holds until the process exits. The call makes no
 * cudaMalloc or cudaFree call and uses no allocating library routine.
 *  - Plans whose usp_ulysses_attention_workspace_size exceeds the array are
 *    rejected with USP_ERR_SHAPE before any launch.
 *  - The array's device address is looked up (cudaGetSymbolAddress) when the
 *    plan is created, with the plan's device current, and kept in the plan; so
 *    the array is reserved on a device no later than the first plan created
 *    there, and this call itself loads nothing. A plan does not outlive the
 *    CUDA context it was created in (after a device reset, create new plans).
 *  - All calls share the one array and it keeps the last call's contents.
 *    Calls that overlap on the GPU (other streams, other host threads, other
 *    plans on the same device) race on it: order them. Nothing in it has to
 *    start at zero.
 */
#define USP_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int usp_ulysses_attention_noalloc(const usp_plan* plan, const void* const* q, const void* const* k,
                                  const void* const* v, void* const* out, float scale, int32_t num_chunks,
                                  void* stream);

/*
 * Rank-local entry points: the Ulysses block across processes, one process
 * (one GPU) per sequence-parallel rank. "h3_blackwell_runtime/distributed.py
 * -- Ragged Ulysses sequence-parallel transport", seq_to_heads / heads_to_seq:
 * each rank packs one contiguous block per peer, the blocks travel in one
 * ragged all-to-all (all_to_all_single with per-peer element counts), and each
 * rank unpacks what it receives in source-rank order. API page,
 * ulysses_attention(prefer_all_gather): the same result through equal-size
 * all-gathers (blocks padded to the longest), which a captured CUDA graph can
 * replay. The library packs, unpacks and computes; the caller runs the
 * collective (e.g. NCCL through torch.distributed) on buffers it owns.
 *
 * Every rank creates the same plan (same sizes, world = number of ranks) on
 * its own device and passes its rank; only plain and grouped-query plans are
 * taken (a Ulysses + Ring plan returns USP_ERR_UNSUPPORTED). Head chunks are
 * usp_head_chunk_ranges(G = H_0, num_chunks); chunk c exchanges, on every
 * rank j, the query heads of j inside the chunk's local window (n_j of them)
 * and the kv heads whose first query head lies there (m_j; m_j = n_j without
 * grouped-query attention).
 *
 * Wire format, in elements of the plan's type (p = prefix rows, T_i = rank i's
 * tokens, T' = p + T; every block is row-major [B][rows][heads][D]):
 *   USP_DIST_SEQ_TO_HEAD  rank r -> peer j: q [B][p+T_r][n_j][D], then, with
 *       ntensors = 3, k and v [B][p+T_r][m_j][D]. Every rank sends its prefix
 *       rows; receivers keep rank 0's.
 *   USP_DIST_HEAD_TO_SEQ  rank r -> peer j: o [B][p+T_j][n_r][D] (the prefix
 *       rows go to every peer).
 *   USP_DIST_GATHER_SEQ   rank r's all-gather block: its q, k, v sequence
 *       shards back to back ([B][p+T_r][H][D], then [B][p+T_r][Hkv][D] twice),
 *       padded to the longest block over ranks (chunk-independent).
 *   USP_DIST_GATHER_HEADS rank r's all-gather block: o [B][T'][n_r][D],
 *       padded to the longest block over ranks.
 * A block's padding is never read.
 */
#define USP_DIST_SEQ_TO_HEAD 0
#define USP_DIST_HEAD_TO_SEQ 1
#define USP_DIST_GATHER_SEQ 2
#define USP_DIST_GATHER_HEADS 3

/*
 * usp_dist_exchange_counts -- the split lists of one exchange for `rank`
 * (transport page, seq_to_heads: input_splits / output_splits), in elements,
 * computed from the sizes alone (no device is needed, so a host-side
 * collective can be planned anywhere). world arrays: send_counts[j] and
 * send_displs[j] for peer j, recv_counts[i] and recv_displs[i] for source i.
 * All-to-all kinds: displacements are the running sums of the counts. Gather
 * kinds: every count is the padded block, send_displs are 0 and
 * recv_displs[i] = i * block (all_gather_into_tensor's layout).
 * Errors: as usp_plan_create_gqa for the sizes; USP_ERR_INVALID_ARG for a rank
 * outside [0, world), an unknown exchange, ntensors other than 1 or 3
 * (q/k/v kinds) or 1 (output kinds), num_chunks < 1 or a chunk outside the
 * head chunks; NULL outputs.
 */
int usp_dist_exchange_counts(int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv, int32_t head_dim,
                             int32_t world, int32_t prefix_tokens, int32_t rank, int32_t exchange, int32_t ntensors,
                             int32_t num_chunks, int32_t chunk, int64_t* send_counts, int64_t* send_displs,
                             int64_t* recv_counts, int64_t* recv_displs);

/*
 * usp_dist_pack -- fills `send` (usp_dist_exchange_counts' send layout) for
 * chunk `chunk` of `num_chunks`:
 *   SEQ_TO_HEAD   in[t] = this rank's sequence shard of q, k, v
 *                 ([B][p+T_r][H or Hkv][D]); ntensors 1 (q) or 3.
 *   HEAD_TO_SEQ   in[0] = this rank's head shard o [B][T'][H_r][D].
 *   GATHER_SEQ    in[t] as SEQ_TO_HEAD (copied whole; the chunk is ignored).
 *   GATHER_HEADS  in[0] as HEAD_TO_SEQ.
 * Device pointers, 16-byte aligned, caller-owned; send must not overlap in.
 * Errors: as usp_dist_exchange_counts, plus USP_ERR_ALIGN and USP_ERR_CUDA.
 */
int usp_dist_pack(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t ntensors, int32_t num_chunks,
                  int32_t chunk, const void* const* in, void* send, void* stream);

/*
 * usp_dist_unpack -- reads `recv` (usp_dist_exchange_counts' receive layout,
 * after the collective) for chunk `chunk` of `num_chunks`:
 *   SEQ_TO_HEAD, GATHER_SEQ  out[t] = this rank's head shards of q, k, v
 *                 [B][T'][H_r or Hkv_r][D]; the chunk's heads are written (all
 *                 chunks in order fill the shards).
 *   HEAD_TO_SEQ, GATHER_HEADS  out[0] = this rank's sequence shard
 *                 [B][p+T_r][H][D]; the chunk's heads of every rank are written.
 * Errors as usp_dist_pack.
 */
int usp_dist_unpack(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t ntensors, int32_t num_chunks,
                    int32_t chunk, const void* recv, void* const* out, void* stream);

/*
 * usp_dist_workspace_size -- bytes of workspace usp_dist_attention needs on
 * `rank`: (H_r + 2 Hkv_r) * B * T' * D elements, each part 256-byte aligned.
 */
int usp_dist_workspace_size(const usp_plan* plan, int32_t rank, size_t* bytes);

/*
 * usp_dist_attention -- API page, ulysses_attention's run_attention on one
 * rank, for the heads of chunk `chunk`: `recv` holds the received q, k, v
 * (exchange USP_DIST_SEQ_TO_HEAD with ntensors 3, or USP_DIST_GATHER_SEQ);
 * they are unpacked into `workspace` and attended (non-causal softmax
 * attention over all T' tokens, as usp_head_attention), and the epilogue
 * writes the output straight into `send_o` in the layout of the way back:
 * USP_DIST_HEAD_TO_SEQ blocks (row t to the block of the peer owning token t)
 * for SEQ_TO_HEAD, or this rank's USP_DIST_GATHER_HEADS block for GATHER_SEQ.
 * scale <= 0 selects 1/sqrt(D). workspace: at least usp_dist_workspace_size()
 * bytes, 256-byte aligned; its contents are scratch, but with grouped-query
 * attention a kv head shared by two chunks arrives with the first of them, so
 * a block's chunks must run in order on the same workspace. Errors as
 * usp_dist_pack, plus those of usp_ulysses_attention's attention.
 */
int usp_dist_attention(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t num_chunks, int32_t chunk,
                       const void* recv, void* send_o, float scale, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * usp_ulysses_attention_graph_create -- captures one usp_ulysses_attention
 * call (its packs, attention launches and the auxiliary-stream chunk
 * overlap) into a CUDA graph owned by the returned handle, without running it.
 * Arguments as usp_ulysses_attention; the buffer pointers are fixed in the
 * graph, so a caller refreshes inputs by writing into the same q/k/v buffers
 * and replays with usp_graph_launch, one launch per block. The plan must
 * outlive the graph only for usp_graph_destroy's bookkeeping: the graph
 * itself holds no reference to the plan's streams or events. Errors as
 * usp_ulysses_attention (nothing is captured then), plus USP_ERR_CUDA if the
 * capture or instantiation fails.
 */
typedef struct usp_graph usp_graph;
int usp_ulysses_attention_graph_create(usp_graph** out, const usp_plan* plan, const void* const* q,
                                       const void* const* k, const void* const* v, void* const* o, float scale,
                                       int32_t num_chunks, void* workspace, size_t workspace_bytes);

/* Launches the captured block on `stream` (a cudaStream_t; NULL = the legacy default stream). */
int usp_graph_launch(usp_graph* graph, void* stream);

/* Releases the graph (NULL is ignored). Launches already enqueued complete normally. */
int usp_graph_destroy(usp_graph* graph);

/*
 * usp_plan_set_timing_events -- profiling hook: while set, every
 * usp_ulysses_attention call with this plan records `start` (a cudaEvent_t)
 * on its stream just before its first attention kernel and `stop` just after
 * its last one, so the caller can time the attention kernels alone inside a
 * longer stream of work. NULL, NULL turns it off. The events stay owned by
 * the caller and must outlive their use.
 */
int usp_plan_set_timing_events(usp_plan* plan, void* start, void* stop);

/* Number of kernels this library has launched in this process (diagnostic). */
uint64_t usp_kernel_launches(void);

/*
 * usp_device_status -- synchronises the current device, then reads the
 * library's device-side error words (0 = no error). A bounded device-side
 * wait that ran out returns USP_ERR_TIMEOUT with *code = the wait's site; in
 * a bounds-checking build (-DUSP_BOUNDS_CHECK), an out-of-range offset that a
 * kernel skipped returns USP_ERR_BOUNDS with *code = the access site. reset
 * != 0 clears the words. Diagnostic only.
 */
int usp_device_status(uint32_t* code, int32_t reset);

/*
 * usp_debug_wait_timeout -- launches one CTA that waits on a barrier nothing
 * arrives on, with a limit of `limit_us` microseconds (1..2000000); the wait
 * gives up, records the error word and returns. Used to test that a wait that
 * runs out reports USP_ERR_TIMEOUT through usp_device_status without faulting
 * or hanging the GPU.
 */
int usp_debug_wait_timeout(uint32_t limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* USP_H_ */
