// Rank-local entry points of the Ulysses block across processes: one process
// (one GPU) per sequence-parallel rank, the exchange itself done by the
// caller's collective library.
//
// "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
// transport", seq_to_heads / heads_to_seq: each rank packs one contiguous
// block per peer, the blocks travel in one ragged all-to-all whose per-peer
// element counts are the split lists, and each rank unpacks the blocks it
// receives in source-rank order. The API page
// "mstar.model.components.distributed.sequence_parallel", ulysses_attention
// (prefer_all_gather), offers the same result through equal-size all-gathers
// (shards padded to the longest): every rank gathers every rank's q/k/v
// sequence shards and keeps its own heads, then gathers every rank's output
// heads and keeps its own tokens.
//
// The wire format (elements of the plan's type; B = batch, p = prefix rows,
// T_i = tokens of rank i, D = head_dim; c = the head chunk, whose heads on rank
// j are n_j query heads and m_j kv heads; "rows" are [B][rows][heads][D]):
//   SEQ_TO_HEAD   rank r -> peer j: q [B][p+T_r][n_j][D], then (3 tensors)
//                 k and v [B][p+T_r][m_j][D]. Every rank sends its prefix
//                 rows; the receiver keeps source 0's.
//   HEAD_TO_SEQ   rank r -> peer j: o [B][p+T_j][n_r][D] (prefix rows to all).
//   GATHER_SEQ    rank r's block: q, k, v sequence shards back to back
//                 ([B][p+T_r][H or Hkv][D]), padded to the longest block.
//   GATHER_HEADS  rank r's block: o [B][T'][n_r][D], padded to the longest.
// Every move is an instance of the layout kernels (TMA tile copies or 16-byte
// vectors); the attention's epilogue writes its output straight into the
// HEAD_TO_SEQ (or GATHER_HEADS) send layout, so the way back needs no pack.
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "usp_internal.h"

namespace {

struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

// Heads of rank j inside head-chunk window [lo, hi) (global numbering): its
// query heads, and the kv heads whose first query head falls in the window
// (so each kv head travels with exactly one chunk).
struct ChunkHeads {
  int32_t q0, nq, kv0, nkv;
};

ChunkHeads chunk_heads(const usp_plan* p, int j, int lo, int hi) {
  ChunkHeads c{};
  const int hl = p->head_len[j];
  c.q0 = p->head_start[j] + lo;
  c.nq = lo < hl ? (hi < hl ? hi : hl) - lo : 0;
  const int g = p->kv_group;
  c.kv0 = (c.q0 + g - 1) / g;
  c.nkv = c.nq > 0 ? (c.q0 + c.nq + g - 1) / g - c.kv0 : 0;
  if (c.nq == 0) c.kv0 = p->kv_head_start[j];
  return c;
}

struct Exchange {
  int32_t lo = 0, hi = 0;  // the chunk's local-head window
  int64_t send_counts[USP_MAX_WORLD] = {}, send_displs[USP_MAX_WORLD] = {};
  int64_t recv_counts[USP_MAX_WORLD] = {}, recv_displs[USP_MAX_WORLD] = {};
};

int check_exchange_args(const usp_plan* p, int32_t rank, int32_t exchange, int32_t ntensors, int32_t num_chunks,
                        int32_t chunk, Exchange* x) {
  if (p->ring > 1)
    return usp::set_error(USP_ERR_UNSUPPORTED, "the rank-local entry points take plain (or grouped-query) plans, not "
                          "a Ulysses + Ring hybrid");
  if (rank < 0 || rank >= p->world)
    return usp::set_error(USP_ERR_INVALID_ARG, "rank %d outside [0, %d)", rank, p->world);
  if (exchange < USP_DIST_SEQ_TO_HEAD || exchange > USP_DIST_GATHER_HEADS)
    return usp::set_error(USP_ERR_INVALID_ARG, "unknown exchange %d", exchange);
  const bool qkv = exchange == USP_DIST_SEQ_TO_HEAD || exchange == USP_DIST_GATHER_SEQ;
  if (qkv ? (ntensors != 1 && ntensors != 3) : ntensors != 1)
    return usp::set_error(USP_ERR_INVALID_ARG, "ntensors must be %s for this exchange (got %d)", qkv ? "1 or 3" : "1",
                          ntensors);
  if (num_chunks < 1) return usp::set_error(USP_ERR_INVALID_ARG, "num_chunks must be positive (got %d)", num_chunks);
  int32_t n = 0, lo[USP_MAX_HEADS], hi[USP_MAX_HEADS];
  usp_head_chunk_ranges(p->group_heads, num_chunks, &n, lo, hi);
  if (chunk < 0 || chunk >= n)
    return usp::set_error(USP_ERR_INVALID_ARG, "chunk %d outside the %d head chunks of num_chunks=%d", chunk, n,
                          num_chunks);
  x->lo = lo[chunk];
  x->hi = hi[chunk];
  return USP_OK;
}

// Per-peer element counts and displacements of one exchange (see the wire
// format above); the caller has checked the arguments.
void exchange_counts(const usp_plan* p, int32_t r, int32_t exchange, int32_t nt, Exchange* x) {
  const int64_t B = p->batch, pre = p->prefix, D = p->head_dim, P = p->world, Tp = p->tokens();
  const ChunkHeads own = chunk_heads(p, r, x->lo, x->hi);
  auto heads_of = [&](const ChunkHeads& c) { return c.nq + (nt == 3 ? 2 * c.nkv : 0); };
  int64_t block = 0;
  switch (exchange) {
    case USP_DIST_SEQ_TO_HEAD:
      for (int j = 0; j < P; ++j) {
        x->send_counts[j] = B * (pre + p->tok_len[r]) * D * heads_of(chunk_heads(p, j, x->lo, x->hi));
        x->recv_counts[j] = B * (pre + p->tok_len[j]) * D * heads_of(own);
      }
      break;
    case USP_DIST_HEAD_TO_SEQ:
      for (int j = 0; j < P; ++j) {
        x->send_counts[j] = B * (pre + p->tok_len[j]) * D * own.nq;
        x->recv_counts[j] = B * (pre + p->tok_len[r]) * D * chunk_heads(p, j, x->lo, x->hi).nq;
      }
      break;
    case USP_DIST_GATHER_SEQ:
      for (int j = 0; j < P; ++j) {
        const int64_t b = B * (pre + p->tok_len[j]) * D * (p->heads + (nt == 3 ? 2 * p->heads_kv : 0));
        block = b > block ? b : block;
      }
      break;
    default:  // USP_DIST_GATHER_HEADS
      for (int j = 0; j < P; ++j) {
        const int64_t b = B * Tp * D * chunk_heads(p, j, x->lo, x->hi).nq;
        block = b > block ? b : block;
      }
      break;
  }
  if (exchange == USP_DIST_GATHER_SEQ || exchange == USP_DIST_GATHER_HEADS) {
    // equal-size all-gather: one padded block from every rank, in rank order
    for (int j = 0; j < P; ++j) {
      x->send_counts[j] = block;
      x->send_displs[j] = 0;
      x->recv_counts[j] = block;
      x->recv_displs[j] = j * block;
    }
    return;
  }
  int64_t s = 0, q = 0;
  for (int j = 0; j < P; ++j) {
    x->send_displs[j] = s;
    x->recv_displs[j] = q;
    s += x->send_counts[j];
    q += x->recv_counts[j];
  }
}

void base_args(usp::PermuteArgs& a, const usp_plan* p, int dir) {
  memset(&a, 0, sizeof(a));
  a.dir = dir;
  a.outer = p->batch;
  a.dv = static_cast<int32_t>(static_cast<int64_t>(p->head_dim) * p->elem / usp::plan_vec_bytes(p));
}

// The sequence side is one buffer of `rows` rows per batch element, row t of
// it being head-side row tok0 + t (no prefix handling).
void one_seq_buffer(usp::PermuteArgs& a, const usp_plan* p, int64_t rows, int64_t tok0) {
  a.n_seq = 1;
  a.prefix = 0;
  a.seq_rows[0] = 0;
  a.seq_rows[1] = p->batch * rows;
  a.tok_start[0] = tok0;
  a.tok_len[0] = rows;
}

// The sequence side is P buffers, buffer i holding the prefix rows and rank
// i's tokens of every batch element (the plan's own sequence-shard layout).
void rank_seq_buffers(usp::PermuteArgs& a, const usp_plan* p) {
  a.n_seq = p->world;
  a.prefix = p->prefix;
  a.seq_rows[0] = 0;
  for (int s = 0; s < p->world; ++s) {
    a.tok_start[s] = p->tok_start[s];
    a.tok_len[s] = p->tok_len[s];
    a.seq_rows[s + 1] = a.seq_rows[s] + p->batch * (p->prefix + p->tok_len[s]);
  }
}

// Selects units [first, first + count) owned by head-side buffer `buf`.
void select_units(usp::PermuteArgs& a, int first, int count, int buf) {
  for (int u = 0; u < count; ++u) {
    a.sel_head[a.nsel] = static_cast<uint16_t>(first + u);
    a.sel_rank[a.nsel] = static_cast<uint8_t>(buf);
    ++a.nsel;
  }
}

uint8_t* at(const void* base, int64_t elems, int elem) {
  return static_cast<uint8_t*>(const_cast<void*>(base)) + elems * elem;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t ws_part(const usp_plan* p, int32_t heads) {
  return align256(static_cast<size_t>(p->batch) * p->tokens() * heads * p->head_dim * p->elem);
}

// Received q/k/v blocks (SEQ_TO_HEAD or GATHER_SEQ layout) -> this rank's head
// shards of the chunk's heads. head_major: [H_r][B][T'][D] (the attention
// workspace) instead of the public [B][T'][H_r][D].
int unpack_qkv(const usp_plan* p, int32_t r, int32_t exchange, int32_t nt, const Exchange& x, const void* recv,
               void* const* out, bool head_major, cudaStream_t stream) {
  const ChunkHeads own = chunk_heads(p, r, x.lo, x.hi);
  if (own.nq == 0) return USP_OK;
  const bool gqa = p->kv_group > 1 && nt == 3;
  for (int part = 0; part < (gqa ? 2 : 1); ++part) {
    const bool kvpart = part == 1;
    usp::PermuteArgs a;
    base_args(a, p, 0);
    rank_seq_buffers(a, p);
    a.ntensors = gqa ? (kvpart ? 2 : 1) : nt;
    a.n_head = 1;
    a.head_layout = head_major ? 1 : 0;
    a.full_tokens = p->tokens();
    a.explicit_counts = 1;
    a.head_start[0] = kvpart ? p->kv_head_start[r] : p->head_start[r];
    a.head_count[0] = kvpart ? p->kv_head_len[r] : p->head_len[r];
    const int first = kvpart ? own.kv0 : own.q0;
    const int count = kvpart ? own.nkv : own.nq;
    if (count == 0) continue;
    select_units(a, first, count, 0);
    const int t_first = gqa ? (kvpart ? 1 : 0) : 0;
    for (int t = 0; t < a.ntensors; ++t) {
      const int tensor = t_first + t;  // 0 q, 1 k, 2 v
      a.head_ptr[t][0] = out[tensor];
      for (int i = 0; i < p->world; ++i) {
        const int64_t rows = p->batch * (p->prefix + p->tok_len[i]);
        int64_t off = x.recv_displs[i];
        if (exchange == USP_DIST_SEQ_TO_HEAD) {
          // this rank's chunk heads only: [n_r rows q][m_r rows k][m_r rows v]
          a.heads = kvpart ? own.nkv : own.nq;
          a.seq_unit_base = first;
          off += rows * p->head_dim * (tensor == 0 ? 0 : own.nq + (tensor == 2 ? own.nkv : 0));
        } else {
          // whole sequence shards: [H rows q][Hkv rows k][Hkv rows v]
          a.heads = kvpart || (!gqa && tensor > 0) ? p->heads_kv : p->heads;
          a.seq_unit_base = 0;
          off += rows * p->head_dim * (tensor == 0 ? 0 : p->heads + (tensor == 2 ? p->heads_kv : 0));
        }
        a.seq_ptr[t][i] = at(recv, off, p->elem);
      }
    }
    if (int rc = usp::plan_launch_pack(p, a, stream)) return rc;
  }
  return USP_OK;
}

int check_rank_call(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t ntensors, int32_t num_chunks,
                    int32_t chunk, Exchange* x) {
  if (!plan) return usp::set_error(USP_ERR_INVALID_ARG, "plan is NULL");
  if (int rc = check_exchange_args(plan, rank, exchange, ntensors, num_chunks, chunk, x)) return rc;
  if (int rc = usp::plan_check_device(plan)) return rc;
  exchange_counts(plan, rank, exchange, ntensors, x);
  return USP_OK;
}

}  // namespace

extern "C" {

int usp_dist_exchange_counts(int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv, int32_t head_dim,
                             int32_t world, int32_t prefix_tokens, int32_t rank, int32_t exchange, int32_t ntensors,
                             int32_t num_chunks, int32_t chunk, int64_t* send_counts, int64_t* send_displs,
                             int64_t* recv_counts, int64_t* recv_displs) {
  if (!send_counts || !send_displs || !recv_counts || !recv_displs)
    return usp::set_error(USP_ERR_INVALID_ARG, "output arrays must not be NULL");
  usp_plan p;
  if (int rc = usp::plan_geometry(&p, batch, seq_len, heads, heads_kv, head_dim, world, 1, USP_BF16, prefix_tokens))
    return rc;
  Exchange x;
  if (int rc = check_exchange_args(&p, rank, exchange, ntensors, num_chunks, chunk, &x)) return rc;
  exchange_counts(&p, rank, exchange, ntensors, &x);
  for (int j = 0; j < world; ++j) {
    send_counts[j] = x.send_counts[j];
    send_displs[j] = x.send_displs[j];
    recv_counts[j] = x.recv_counts[j];
    recv_displs[j] = x.recv_displs[j];
  }
  return USP_OK;
}

int usp_dist_workspace_size(const usp_plan* plan, int32_t rank, size_t* bytes) {
  if (!plan) return usp::set_error(USP_ERR_INVALID_ARG, "plan is NULL");
  if (!bytes) return usp::set_error(USP_ERR_INVALID_ARG, "bytes is NULL");
  if (rank < 0 || rank >= plan->world)
    return usp::set_error(USP_ERR_INVALID_ARG, "rank %d outside [0, %d)", rank, plan->world);
  *bytes = ws_part(plan, plan->head_len[rank]) + 2 * ws_part(plan, plan->kv_head_len[rank]);
  return USP_OK;
}

int usp_dist_pack(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t ntensors, int32_t num_chunks,
                  int32_t chunk, const void* const* in, void* send, void* stream) {
  Range range("usp_dist_pack");
  Exchange x;
  if (int rc = check_rank_call(plan, rank, exchange, ntensors, num_chunks, chunk, &x)) return rc;
  if (!in) return usp::set_error(USP_ERR_INVALID_ARG, "in is NULL");
  for (int t = 0; t < ntensors; ++t)
    if (int rc = usp::plan_check_ptr(in[t], "in[t]")) return rc;
  if (int rc = usp::plan_check_ptr(send, "send")) return rc;
  const usp_plan* p = plan;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int r = rank;
  const ChunkHeads own = chunk_heads(p, r, x.lo, x.hi);
  if (exchange == USP_DIST_GATHER_SEQ) {
    // the whole sequence shards, back to back (the padding is never read)
    const int64_t rows = p->batch * (p->prefix + p->tok_len[r]);
    int64_t off = 0;
    for (int t = 0; t < ntensors; ++t) {
      const int64_t n = rows * (t == 0 ? p->heads : p->heads_kv) * p->head_dim;
      if (int rc = usp::cuda_check(cudaMemcpyAsync(at(send, off, p->elem), in[t], n * p->elem,
                                                   cudaMemcpyDeviceToDevice, s), "cudaMemcpyAsync(gather block)"))
        return rc;
      off += n;
    }
    return USP_OK;
  }
  if (exchange == USP_DIST_SEQ_TO_HEAD) {
    const bool gqa = p->kv_group > 1 && ntensors == 3;
    for (int part = 0; part < (gqa ? 2 : 1); ++part) {
      const bool kvpart = part == 1;
      usp::PermuteArgs a;
      base_args(a, p, 0);
      one_seq_buffer(a, p, p->prefix + p->tok_len[r], 0);
      a.ntensors = gqa ? (kvpart ? 2 : 1) : ntensors;
      a.heads = kvpart ? p->heads_kv : p->heads;
      a.n_head = p->world;
      a.head_layout = 0;
      a.full_tokens = p->prefix + p->tok_len[r];
      a.explicit_counts = 1;
      for (int j = 0; j < p->world; ++j) {
        const ChunkHeads cj = chunk_heads(p, j, x.lo, x.hi);
        a.head_start[j] = kvpart ? cj.kv0 : cj.q0;
        a.head_count[j] = kvpart ? cj.nkv : cj.nq;
        select_units(a, a.head_start[j], a.head_count[j], j);
      }
      if (a.nsel == 0) continue;
      const int t_first = gqa ? (kvpart ? 1 : 0) : 0;
      const int64_t rows = p->batch * (p->prefix + p->tok_len[r]);
      for (int t = 0; t < a.ntensors; ++t) {
        const int tensor = t_first + t;
        a.seq_ptr[t][0] = const_cast<void*>(in[tensor]);
        for (int j = 0; j < p->world; ++j) {
          const ChunkHeads cj = chunk_heads(p, j, x.lo, x.hi);
          const int64_t off = x.send_displs[j] + rows * p->head_dim * (tensor == 0 ? 0 : cj.nq + (tensor == 2 ? cj.nkv : 0));
          a.head_ptr[t][j] = at(send, off, p->elem);
        }
      }
      if (int rc = usp::plan_launch_pack(p, a, s)) return rc;
    }
    return USP_OK;
  }
  if (own.nq == 0) return USP_OK;
  usp::PermuteArgs a;
  if (exchange == USP_DIST_HEAD_TO_SEQ) {
    // this rank's head shard o [B][T'][H_r][D] -> per-peer row blocks of the chunk's heads
    base_args(a, p, 1);
    rank_seq_buffers(a, p);
    a.ntensors = 1;
    a.heads = own.nq;
    a.seq_unit_base = own.q0;
    for (int j = 0; j < p->world; ++j) a.seq_ptr[0][j] = at(send, x.send_displs[j], p->elem);
  } else {  // USP_DIST_GATHER_HEADS: the chunk's heads of o, [B][T'][n_r][D]
    base_args(a, p, 0);
    one_seq_buffer(a, p, p->tokens(), 0);
    a.ntensors = 1;
    a.heads = p->head_len[r];
    a.seq_unit_base = p->head_start[r];
    a.seq_ptr[0][0] = const_cast<void*>(in[0]);
  }
  a.n_head = 1;
  a.head_layout = 0;
  a.full_tokens = p->tokens();
  a.explicit_counts = 1;
  if (exchange == USP_DIST_HEAD_TO_SEQ) {
    a.head_start[0] = p->head_start[r];
    a.head_count[0] = p->head_len[r];
    a.head_ptr[0][0] = const_cast<void*>(in[0]);
  } else {
    a.head_start[0] = own.q0;
    a.head_count[0] = own.nq;
    a.head_ptr[0][0] = send;
  }
  select_units(a, own.q0, own.nq, 0);
  return usp::plan_launch_pack(p, a, s);
}

int usp_dist_unpack(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t ntensors, int32_t num_chunks,
                    int32_t chunk, const void* recv, void* const* out, void* stream) {
  Range range("usp_dist_unpack");
  Exchange x;
  if (int rc = check_rank_call(plan, rank, exchange, ntensors, num_chunks, chunk, &x)) return rc;
  if (int rc = usp::plan_check_ptr(recv, "recv")) return rc;
  if (!out) return usp::set_error(USP_ERR_INVALID_ARG, "out is NULL");
  for (int t = 0; t < ntensors; ++t)
    if (int rc = usp::plan_check_ptr(out[t], "out[t]")) return rc;
  const usp_plan* p = plan;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int r = rank;
  if (exchange == USP_DIST_SEQ_TO_HEAD || exchange == USP_DIST_GATHER_SEQ)
    return unpack_qkv(p, r, exchange, ntensors, x, recv, out, false, s);
  // HEAD_TO_SEQ / GATHER_HEADS: every rank's chunk heads -> this rank's sequence shard
  usp::PermuteArgs a;
  base_args(a, p, 1);
  if (exchange == USP_DIST_HEAD_TO_SEQ) {
    one_seq_buffer(a, p, p->prefix + p->tok_len[r], 0);
    a.full_tokens = p->prefix + p->tok_len[r];
  } else {
    // rows: the prefix rows, then this rank's tokens, of the full sequence
    a.n_seq = 1;
    a.prefix = p->prefix;
    a.seq_rows[0] = 0;
    a.seq_rows[1] = p->batch * (p->prefix + p->tok_len[r]);
    a.tok_start[0] = p->tok_start[r];
    a.tok_len[0] = p->tok_len[r];
    a.full_tokens = p->tokens();
  }
  a.ntensors = 1;
  a.heads = p->heads;
  a.n_head = p->world;
  a.head_layout = 0;
  a.explicit_counts = 1;
  a.seq_ptr[0][0] = out[0];
  for (int i = 0; i < p->world; ++i) {
    const ChunkHeads ci = chunk_heads(p, i, x.lo, x.hi);
    a.head_start[i] = ci.q0;
    a.head_count[i] = ci.nq;
    a.head_ptr[0][i] = at(recv, x.recv_displs[i], p->elem);
    select_units(a, ci.q0, ci.nq, i);
  }
  if (a.nsel == 0) return USP_OK;
  return usp::plan_launch_pack(p, a, s);
}

int usp_dist_attention(const usp_plan* plan, int32_t rank, int32_t exchange, int32_t num_chunks, int32_t chunk,
                       const void* recv, void* send_o, float scale, void* workspace, size_t workspace_bytes,
                       void* stream) {
  Range range("usp_dist_attention");
  if (exchange != USP_DIST_SEQ_TO_HEAD && exchange != USP_DIST_GATHER_SEQ)
    return usp::set_error(USP_ERR_INVALID_ARG, "usp_dist_attention takes received q/k/v of USP_DIST_SEQ_TO_HEAD or "
                          "USP_DIST_GATHER_SEQ (got %d)", exchange);
  Exchange x;
  if (int rc = check_rank_call(plan, rank, exchange, 3, num_chunks, chunk, &x)) return rc;
  if (int rc = usp::plan_check_ptr(recv, "recv")) return rc;
  if (int rc = usp::plan_check_ptr(send_o, "send_o")) return rc;
  if (!workspace) return usp::set_error(USP_ERR_INVALID_ARG, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return usp::set_error(USP_ERR_ALIGN, "workspace must be 256-byte aligned");
  size_t need = 0;
  usp_dist_workspace_size(plan, rank, &need);
  if (workspace_bytes < need)
    return usp::set_error(USP_ERR_SHAPE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  if (int rc = usp::plan_check_attention(plan)) return rc;
  const usp_plan* p = plan;
  const int r = rank;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ChunkHeads own = chunk_heads(p, r, x.lo, x.hi);
  if (own.nq == 0) return USP_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* parts[3] = {ws, ws + ws_part(p, p->head_len[r]),
                    ws + ws_part(p, p->head_len[r]) + ws_part(p, p->kv_head_len[r])};
  if (int rc = unpack_qkv(p, r, exchange, 3, x, recv, parts, true, s)) return rc;

  const int64_t B = p->batch, T = p->tokens(), D = p->head_dim;
  usp::AttnLaunch L;
  memset(&L, 0, sizeof(L));
  L.in.q = parts[0];
  L.in.k = parts[1];
  L.in.v = parts[2];
  L.in.qv = {B * T * D, D, T * D, p->head_len[r]};
  L.in.kvv = {B * T * D, D, T * D, p->kv_head_len[r]};
  L.in.kv_group = p->kv_group;
  L.in.q_head_base = p->head_start[r];
  L.in.kv_head_base = p->kv_head_start[r];
  L.out.out_heads = own.nq;
  L.out.head_base = x.lo;
  if (exchange == USP_DIST_SEQ_TO_HEAD) {
    // the epilogue writes each row into the HEAD_TO_SEQ block of the peer owning its token
    Exchange back;
    back.lo = x.lo;
    back.hi = x.hi;
    exchange_counts(p, r, USP_DIST_HEAD_TO_SEQ, 1, &back);
    L.out.nseg = p->world;
    L.out.prefix = p->prefix;
    for (int j = 0; j < p->world; ++j) {
      L.out.seg_start[j] = p->tok_start[j];
      L.out.seg_len[j] = p->tok_len[j];
      L.out.seg_ptr[j] = at(send_o, back.send_displs[j], p->elem);
    }
  } else {
    // GATHER_HEADS block: [B][T'][n_r][D]
    L.out.nseg = 1;
    L.out.prefix = 0;
    L.out.seg_start[0] = 0;
    L.out.seg_len[0] = T;
    L.out.seg_ptr[0] = send_o;
  }
  L.tokens = static_cast<int32_t>(T);
  L.batch = static_cast<int32_t>(B);
  L.head_dim = static_cast<int32_t>(D);
  L.dtype = p->dtype;
  L.scale = usp::plan_scale(p, scale);
  L.max_ctas = p->attn_ctas;
  L.kernel = p->attn_kernel;
  L.n_heads = own.nq;
  for (int i = 0; i < own.nq; ++i) L.heads[i] = static_cast<uint16_t>(x.lo + i);
  return usp::plan_launch_attention(L, s);
}

}  // extern "C"
