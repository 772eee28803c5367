// C ABI of libusp: plan (ragged token/head ownership of P virtual ranks),
// argument checking, and the launch sequence of every entry point.
//
// Ownership and splits follow "h3_blackwell_runtime/distributed.py -- Ragged
// Ulysses sequence-parallel transport" (balanced_ranges,
// SequenceParallelContext); the entry points follow the API page
// "mstar.model.components.distributed.sequence_parallel"; head chunks follow
// "maxdiffusion PR #428: experimental two-phase (head-chunked) Ulysses
// all-to-all"; the replicated cls prefix follows "deepspeed/sequence/autosp_vit.py".
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "usp_internal.h"

namespace {

thread_local std::string g_last_error;

// NVTX range over one host call or step (the CPU side of a profiler timeline;
// free when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(int dtype) {
  switch (dtype) {
    case USP_BF16:
    case USP_FP16: return 2;
    case USP_FP32: return 4;
    default: return 0;
  }
}

// Balanced contiguous non-empty split: the first total % parts ranges take one more.
int balanced(int64_t total, int32_t parts, int64_t* starts, int64_t* lengths) {
  if (parts < 1) return usp::set_error(USP_ERR_INVALID_ARG, "parts must be positive (got %d)", parts);
  if (total < parts)
    return usp::set_error(USP_ERR_INVALID_ARG, "cannot split %lld items into %d non-empty ranges",
                          static_cast<long long>(total), parts);
  const int64_t base = total / parts, extra = total % parts;
  int64_t start = 0;
  for (int32_t r = 0; r < parts; ++r) {
    const int64_t len = base + (r < extra ? 1 : 0);
    if (starts) starts[r] = start;
    if (lengths) lengths[r] = len;
    start += len;
  }
  return USP_OK;
}

int check_plan(const usp_plan* plan) {
  if (!plan) return usp::set_error(USP_ERR_INVALID_ARG, "plan is NULL");
  return USP_OK;
}

int check_ptrs(const void* const* ptrs, int n, const char* what) {
  if (!ptrs) return usp::set_error(USP_ERR_INVALID_ARG, "%s: pointer array is NULL", what);
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) return usp::set_error(USP_ERR_INVALID_ARG, "%s[%d] is NULL", what, i);
    if (!aligned16(ptrs[i])) return usp::set_error(USP_ERR_ALIGN, "%s[%d] is not 16-byte aligned", what, i);
  }
  return USP_OK;
}

// Per-rank head shards exist only in the plain block (one head range per rank).
int check_flat(const usp_plan* plan, const char* what) {
  if (plan->ring > 1)
    return usp::set_error(USP_ERR_UNSUPPORTED, "%s: the plan is a Ulysses + Ring hybrid; its head shards are "
                          "internal to usp_ulysses_attention", what);
  return USP_OK;
}

int check_ptr(const void* p, const char* what) {
  if (!p) return usp::set_error(USP_ERR_INVALID_ARG, "%s is NULL", what);
  if (!aligned16(p)) return usp::set_error(USP_ERR_ALIGN, "%s is not 16-byte aligned", what);
  return USP_OK;
}

// Largest vector width (16/8/4/2 bytes) dividing the head-unit size.
int pick_vec(int64_t unit_bytes) {
  for (int v : {16, 8, 4, 2})
    if (unit_bytes % v == 0) return v;
  return 0;
}

int device_matches(const usp_plan* plan) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return usp::cuda_check(e, "cudaGetDevice");
  if (dev != plan->device)
    return usp::set_error(USP_ERR_INVALID_ARG, "plan was created on device %d but device %d is current", plan->device,
                          dev);
  return USP_OK;
}

// Fills the parts of PermuteArgs that describe the plan's ranks.
void fill_seq_side(usp::PermuteArgs& a, const usp_plan* p, int64_t outer) {
  a.n_seq = p->world;
  a.prefix = p->prefix;
  a.outer = outer;
  a.seq_rows[0] = 0;
  for (int s = 0; s < p->world; ++s) {
    a.tok_start[s] = p->tok_start[s];
    a.tok_len[s] = p->tok_len[s];
    a.seq_rows[s + 1] = a.seq_rows[s] + outer * (p->prefix + p->tok_len[s]);
  }
}

void select_all_heads(usp::PermuteArgs& a, int heads, const int32_t* head_start, int nranks) {
  a.nsel = heads;
  int r = 0;
  for (int h = 0; h < heads; ++h) {
    while (r + 1 < nranks && h >= head_start[r + 1]) ++r;
    a.sel_head[h] = static_cast<uint16_t>(h);
    a.sel_rank[h] = static_cast<uint8_t>(r);
  }
}

// Heads of local window [lo, hi) on every rank (ragged: clipped to H_r).
void select_chunk_heads(usp::PermuteArgs& a, const usp_plan* p, int lo, int hi) {
  a.nsel = 0;
  for (int r = 0; r < p->head_ranks; ++r)
    for (int h = lo; h < hi && h < p->head_len[r]; ++h) {
      a.sel_head[a.nsel] = static_cast<uint16_t>(p->head_start[r] + h);
      a.sel_rank[a.nsel] = static_cast<uint8_t>(r);
      ++a.nsel;
    }
}

// A sequence <-> head move: TMA tile copies when the plan asks for them and the
// head unit allows it (a multiple of 16 bytes), else 16-byte vector copies.
// (The TMA launcher counts rows in 32 bits.) Head -> sequence by TMA needs
// every head selected: the replicated prefix rows are then copied whole from
// rank 0's shard to the others.
int launch_pack(const usp_plan* plan, const usp::PermuteArgs& a, int vec, int64_t unit, cudaStream_t stream) {
  const bool tma = plan->pack_mode == USP_PACK_TMA && usp::pack_tma_supported(plan->elem, unit) &&
                   a.seq_rows[a.n_seq] <= INT32_MAX && (a.dir == 0 || a.nsel == a.heads) &&
                   (a.prefix == 0 || a.tok_start[0] == 0);
  if (!tma) return usp::launch_permute(a, vec, stream);
  if (int rc = usp::launch_pack_tma(a, plan->elem, unit, stream)) return rc;
  if (a.dir == 0 || a.prefix == 0 || a.n_seq < 2) return USP_OK;
  for (int t = 0; t < a.ntensors; ++t) {
    usp::CopyArgs c;
    memset(&c, 0, sizeof(c));
    c.to_shards = 1;
    c.outer = a.outer;
    c.nv = a.heads * unit / 16;
    c.full_rows = a.prefix + a.tok_len[0];
    c.full = a.seq_ptr[t][0];
    for (int s = 1; s < a.n_seq; ++s) {
      const int k = s - 1;
      c.shards[s] = a.seq_ptr[t][s];
      c.shard[k] = s;
      c.shard_rows[k] = a.prefix + a.tok_len[s];
      c.srow0[k] = 0;
      c.frow0[k] = 0;
      c.rows[k] = a.prefix;
    }
    c.nkinds = a.n_seq - 1;
    if (int rc = usp::launch_copy_rows(c, stream)) return rc;
  }
  return USP_OK;
}

// kv selects the k/v head geometry (Hkv heads split by kv_head_start) instead
// of the query geometry.
int seq_head_exchange(const usp_plan* plan, int dir, int32_t ntensors, const void* const* seq, void* const* heads,
                      cudaStream_t stream, bool kv = false) {
  const int32_t nheads = kv ? plan->heads_kv : plan->heads;
  const int32_t* hstart = kv ? plan->kv_head_start : plan->head_start;
  usp::PermuteArgs a;
  memset(&a, 0, sizeof(a));
  const int64_t unit = static_cast<int64_t>(plan->head_dim) * plan->elem;
  const int vec = pick_vec(unit);
  a.dir = dir;
  fill_seq_side(a, plan, plan->batch);
  a.n_head = plan->world;
  a.ntensors = ntensors;
  a.heads = nheads;
  a.dv = static_cast<int32_t>(unit / vec);
  a.head_layout = 0;
  a.full_tokens = plan->tokens();
  for (int r = 0; r <= plan->world; ++r) a.head_start[r] = hstart[r];
  select_all_heads(a, nheads, hstart, plan->world);
  for (int t = 0; t < ntensors; ++t)
    for (int r = 0; r < plan->world; ++r) {
      a.seq_ptr[t][r] = const_cast<void*>(seq[t * plan->world + r]);
      a.head_ptr[t][r] = heads[t * plan->world + r];
    }
  return launch_pack(plan, a, vec, unit, stream);
}

}  // namespace

namespace usp {

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

static std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return USP_OK;
  return set_error(USP_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int ensure_smem_limit(const void* func, size_t bytes, const char* what, int carveout) {
  static std::mutex m;
  static std::map<std::pair<const void*, int>, size_t> limits;
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  std::lock_guard<std::mutex> guard(m);
  size_t& set = limits[{func, dev}];
  if (bytes <= set) return USP_OK;
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return cuda_check(e, what);
  if (carveout >= 0) {
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, carveout);
    if (e != cudaSuccess) return cuda_check(e, what);
  }
  set = bytes;
  return USP_OK;
}

}  // namespace usp

namespace usp {

// The plan's device-free part: sizes, the balanced token and head splits and
// the grouped-query check. Fills *p; returns a status (the message is set).
int plan_geometry(usp_plan* p, int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv, int32_t head_dim,
                  int32_t ulysses_size, int32_t ring_size, int32_t dtype, int32_t prefix_tokens) {
  if (ulysses_size < 1 || ring_size < 1 || static_cast<int64_t>(ulysses_size) * ring_size > USP_MAX_WORLD)
    return usp::set_error(USP_ERR_INVALID_ARG, "ulysses_size * ring_size must be in [1, %d] (got %d x %d)",
                          USP_MAX_WORLD, ulysses_size, ring_size);
  const int32_t world = ulysses_size * ring_size;
  const int32_t hr = ulysses_size;  // head ranks
  if (batch < 1) return usp::set_error(USP_ERR_INVALID_ARG, "batch must be positive");
  if (head_dim < 1) return usp::set_error(USP_ERR_INVALID_ARG, "head_dim must be positive");
  if (heads > USP_MAX_HEADS) return usp::set_error(USP_ERR_INVALID_ARG, "heads must be <= %d", USP_MAX_HEADS);
  if (prefix_tokens != 0 && prefix_tokens != 1)
    return usp::set_error(USP_ERR_INVALID_ARG, "prefix_tokens must be 0 or 1 (got %d)", prefix_tokens);
  const int e = elem_bytes(dtype);
  if (!e) return usp::set_error(USP_ERR_DTYPE, "unknown dtype %d", dtype);
  p->batch = batch;
  p->seq_len = seq_len;
  p->heads = heads;
  p->head_dim = head_dim;
  p->world = world;
  p->dtype = dtype;
  p->prefix = prefix_tokens;
  p->elem = e;
  p->head_ranks = hr;
  p->ring = ring_size;
  int rc = balanced(seq_len, world, p->tok_start, p->tok_len);
  if (rc == USP_OK) {
    int64_t hs[USP_MAX_WORLD], hl[USP_MAX_WORLD];
    rc = balanced(heads, hr, hs, hl);
    if (rc == USP_OK) {
      for (int r = 0; r < hr; ++r) {
        p->head_start[r] = static_cast<int32_t>(hs[r]);
        p->head_len[r] = static_cast<int32_t>(hl[r]);
      }
      p->head_start[hr] = heads;
      p->group_heads = p->head_len[0];
    }
  }
  // Grouped-query attention: kv heads split the same way; every rank must own
  // the kv heads its query heads use (query head h uses kv head h / group).
  if (rc == USP_OK) {
    if (heads_kv < 1 || heads % heads_kv != 0)
      rc = usp::set_error(USP_ERR_INVALID_ARG, "query heads (%d) must be a positive multiple of kv heads (%d)", heads,
                          heads_kv);
  }
  if (rc == USP_OK) {
    int64_t ks[USP_MAX_WORLD], kl[USP_MAX_WORLD];
    rc = balanced(heads_kv, hr, ks, kl);
    if (rc == USP_OK) {
      p->heads_kv = heads_kv;
      p->kv_group = heads / heads_kv;
      for (int r = 0; r < hr; ++r) {
        p->kv_head_start[r] = static_cast<int32_t>(ks[r]);
        p->kv_head_len[r] = static_cast<int32_t>(kl[r]);
      }
      p->kv_head_start[hr] = heads_kv;
      for (int r = 0; rc == USP_OK && r < hr; ++r)
        for (int h = p->head_start[r]; h < p->head_start[r + 1]; ++h) {
          const int kvh = h / p->kv_group;
          if (kvh < p->kv_head_start[r] || kvh >= p->kv_head_start[r + 1]) {
            rc = usp::set_error(USP_ERR_SHAPE,
                                "rank %d: query head %d uses kv head %d, outside its kv heads [%d, %d); choose "
                                "head counts whose split keeps each group on one rank (e.g. both divisible by world)",
                                r, h, kvh, p->kv_head_start[r], p->kv_head_start[r + 1]);
            break;
          }
        }
    }
  }
  return rc;
}

}  // namespace usp

extern "C" {

const char* usp_last_error_message(void) { return g_last_error.c_str(); }

int usp_version(void) { return 100; }

int usp_balanced_ranges(int64_t total, int32_t parts, int64_t* starts, int64_t* lengths) {
  if (!starts || !lengths) return usp::set_error(USP_ERR_INVALID_ARG, "output arrays must not be NULL");
  return balanced(total, parts, starts, lengths);
}

int usp_seq_split(int64_t total, int32_t world, int64_t* out_counts) {
  if (!out_counts) return usp::set_error(USP_ERR_INVALID_ARG, "out_counts is NULL");
  return balanced(total, world, nullptr, out_counts);
}

int usp_head_chunk_ranges(int32_t group_heads, int32_t num_chunks, int32_t* n_out, int32_t* lo, int32_t* hi) {
  if (!n_out || !lo || !hi) return usp::set_error(USP_ERR_INVALID_ARG, "output pointers must not be NULL");
  if (group_heads < 1) return usp::set_error(USP_ERR_INVALID_ARG, "group_heads must be positive");
  if (num_chunks < 1) return usp::set_error(USP_ERR_INVALID_ARG, "num_chunks must be positive");
  const int32_t size = (group_heads + num_chunks - 1) / num_chunks;
  int32_t n = 0;
  for (int32_t a = 0; a < group_heads; a += size, ++n) {
    lo[n] = a;
    hi[n] = a + size < group_heads ? a + size : group_heads;
  }
  *n_out = n;
  return USP_OK;
}

int usp_plan_create(usp_plan** out, int64_t batch, int64_t seq_len, int32_t heads, int32_t head_dim, int32_t world,
                    int32_t dtype, int32_t prefix_tokens) {
  return usp_plan_create_hybrid(out, batch, seq_len, heads, heads, head_dim, world, 1, dtype, prefix_tokens);
}

int usp_plan_create_gqa(usp_plan** out, int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv,
                        int32_t head_dim, int32_t world, int32_t dtype, int32_t prefix_tokens) {
  return usp_plan_create_hybrid(out, batch, seq_len, heads, heads_kv, head_dim, world, 1, dtype, prefix_tokens);
}

int usp_plan_create_hybrid(usp_plan** out, int64_t batch, int64_t seq_len, int32_t heads, int32_t heads_kv,
                           int32_t head_dim, int32_t ulysses_size, int32_t ring_size, int32_t dtype,
                           int32_t prefix_tokens) {
  if (!out) return usp::set_error(USP_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  usp_plan* p = new usp_plan();
  int rc = usp::plan_geometry(p, batch, seq_len, heads, heads_kv, head_dim, ulysses_size, ring_size, dtype,
                              prefix_tokens);
  if (rc != USP_OK) {
    delete p;
    return rc;
  }
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    delete p;
    return usp::set_error(USP_ERR_NO_DEVICE, "no CUDA device is visible");
  }
  cudaError_t ce = cudaGetDevice(&p->device);
  if (ce == cudaSuccess) {
    // The allocation-free entry point's scratch address, looked up here so that
    // the call itself never loads a module or touches the runtime's symbol table.
    if (int src = usp::noalloc_scratch_lookup(&p->noalloc_scratch)) {
      usp_plan_destroy(p);
      return src;
    }
    ce = cudaStreamCreateWithFlags(&p->aux, cudaStreamNonBlocking);
  }
  if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&p->ev_inputs, cudaEventDisableTiming);
  for (int c = 0; ce == cudaSuccess && c < p->group_heads; ++c) {
    cudaEvent_t ev;
    ce = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (ce == cudaSuccess) p->ev_chunk.push_back(ev);
  }
  if (ce != cudaSuccess) {
    rc = usp::cuda_check(ce, "plan stream/event creation");
    usp_plan_destroy(p);
    return rc;
  }
  *out = p;
  return USP_OK;
}

int usp_plan_destroy(usp_plan* plan) {
  if (!plan) return USP_OK;
  if (plan->aux) {
    cudaStreamSynchronize(plan->aux);
    cudaStreamDestroy(plan->aux);
  }
  if (plan->ev_inputs) cudaEventDestroy(plan->ev_inputs);
  for (cudaEvent_t ev : plan->ev_chunk) cudaEventDestroy(ev);
  delete plan;
  return USP_OK;
}

int usp_plan_query_kv(const usp_plan* plan, int32_t* heads_kv, int32_t* kv_head_start, int32_t* kv_head_len) {
  if (int rc = check_plan(plan)) return rc;
  if (heads_kv) *heads_kv = plan->heads_kv;
  for (int r = 0; r < plan->world; ++r) {
    const int u = r % plan->head_ranks;  // rank r's position in its Ulysses group
    if (kv_head_start) kv_head_start[r] = plan->kv_head_start[u];
    if (kv_head_len) kv_head_len[r] = plan->kv_head_len[u];
  }
  return USP_OK;
}

int usp_plan_query_hybrid(const usp_plan* plan, int32_t* ulysses_size, int32_t* ring_size) {
  if (int rc = check_plan(plan)) return rc;
  if (ulysses_size) *ulysses_size = plan->head_ranks;
  if (ring_size) *ring_size = plan->ring;
  return USP_OK;
}

int usp_plan_query(const usp_plan* plan, int64_t* tok_start, int64_t* tok_len, int32_t* head_start,
                   int32_t* head_len) {
  if (int rc = check_plan(plan)) return rc;
  for (int r = 0; r < plan->world; ++r) {
    if (tok_start) tok_start[r] = plan->tok_start[r];
    if (tok_len) tok_len[r] = plan->tok_len[r];
    const int u = r % plan->head_ranks;  // rank r's position in its Ulysses group
    if (head_start) head_start[r] = plan->head_start[u];
    if (head_len) head_len[r] = plan->head_len[u];
  }
  return USP_OK;
}

// scatter: the full tensor is the head side with a single head unit per row.
static int scatter_gather(const usp_plan* plan, int dir, const void* full, void* const* shards, int64_t outer,
                          int64_t row_bytes, cudaStream_t stream) {
  if (outer == 0) outer = plan->batch;
  if (row_bytes == 0) row_bytes = static_cast<int64_t>(plan->heads) * plan->head_dim * plan->elem;
  if (outer < 1 || row_bytes < 1) return usp::set_error(USP_ERR_SHAPE, "outer and row_bytes must be positive");
  if (row_bytes % 16 != 0) return usp::set_error(USP_ERR_ALIGN, "row_bytes must be a multiple of 16");
  // Every rank's token window is one contiguous run of rows per batch element
  // in both buffers; the prefix rows go to every shard (scatter) or come from
  // rank 0's (gather).
  usp::CopyArgs a;
  memset(&a, 0, sizeof(a));
  a.to_shards = dir;
  a.outer = outer;
  a.nv = row_bytes / 16;
  a.full_rows = plan->tokens();
  a.full = const_cast<void*>(full);
  const int64_t pre = plan->prefix;
  int n = 0;
  for (int r = 0; r < plan->world; ++r) {
    a.shards[r] = shards[r];
    a.shard[n] = r;
    a.shard_rows[n] = pre + plan->tok_len[r];
    a.srow0[n] = pre;
    a.frow0[n] = pre + plan->tok_start[r];
    a.rows[n] = plan->tok_len[r];
    ++n;
  }
  if (pre > 0) {
    for (int r = 0; r < (dir == 1 ? plan->world : 1); ++r) {
      a.shard[n] = r;
      a.shard_rows[n] = pre + plan->tok_len[r];
      a.srow0[n] = 0;
      a.frow0[n] = 0;
      a.rows[n] = pre;
      ++n;
    }
  }
  a.nkinds = n;
  return usp::launch_copy_rows(a, stream);
}

int usp_scatter_sequence(const usp_plan* plan, const void* x_full, void* const* x_shards, int64_t outer,
                         int64_t row_bytes, void* stream) {
  NvtxRange range("usp_scatter_sequence");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_ptr(x_full, "x_full")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(x_shards), plan->world, "x_shards")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return scatter_gather(plan, 1, x_full, x_shards, outer, row_bytes, static_cast<cudaStream_t>(stream));
}

int usp_gather_sequence(const usp_plan* plan, const void* const* x_shards, void* x_full, int64_t outer,
                        int64_t row_bytes, void* stream) {
  NvtxRange range("usp_gather_sequence");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_ptr(x_full, "x_full")) return rc;
  if (int rc = check_ptrs(x_shards, plan->world, "x_shards")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return scatter_gather(plan, 0, x_full, const_cast<void* const*>(x_shards), outer, row_bytes,
                        static_cast<cudaStream_t>(stream));
}

// head slice: the full tensor is a single sequence-side buffer of `rows` rows.
static int head_slice_gather(const usp_plan* plan, int dir, const void* full, void* const* shards, int64_t rows,
                             cudaStream_t stream) {
  if (rows == 0) rows = plan->batch * plan->tokens();
  if (rows < 1) return usp::set_error(USP_ERR_SHAPE, "rows must be positive");
  const int64_t unit = static_cast<int64_t>(plan->head_dim) * plan->elem;
  const int vec = pick_vec(unit);
  usp::PermuteArgs a;
  memset(&a, 0, sizeof(a));
  a.dir = dir;
  a.n_seq = 1;
  a.prefix = 0;
  a.outer = 1;
  a.seq_rows[0] = 0;
  a.seq_rows[1] = rows;
  a.tok_start[0] = 0;
  a.tok_len[0] = rows;
  a.n_head = plan->world;
  a.ntensors = 1;
  a.heads = plan->heads;
  a.dv = static_cast<int32_t>(unit / vec);
  a.head_layout = 0;
  a.full_tokens = rows;
  for (int r = 0; r <= plan->world; ++r) a.head_start[r] = plan->head_start[r];
  select_all_heads(a, plan->heads, plan->head_start, plan->world);
  a.seq_ptr[0][0] = const_cast<void*>(full);
  for (int r = 0; r < plan->world; ++r) a.head_ptr[0][r] = shards[r];
  // The slice is a sequence -> head move and the gather its inverse (one
  // sequence-side buffer holding every row).
  return launch_pack(plan, a, vec, unit, stream);
}

int usp_sp_head_slice(const usp_plan* plan, const void* x_full, void* const* x_head_shards, int64_t rows,
                      void* stream) {
  NvtxRange range("usp_sp_head_slice");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_flat(plan, "usp_sp_head_slice")) return rc;
  if (int rc = check_ptr(x_full, "x_full")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(x_head_shards), plan->world, "x_head_shards")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return head_slice_gather(plan, 0, x_full, x_head_shards, rows, static_cast<cudaStream_t>(stream));
}

int usp_sp_head_gather(const usp_plan* plan, const void* const* x_head_shards, void* x_full, int64_t rows,
                       void* stream) {
  NvtxRange range("usp_sp_head_gather");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_flat(plan, "usp_sp_head_gather")) return rc;
  if (int rc = check_ptr(x_full, "x_full")) return rc;
  if (int rc = check_ptrs(x_head_shards, plan->world, "x_head_shards")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return head_slice_gather(plan, 1, x_full, const_cast<void* const*>(x_head_shards), rows,
                           static_cast<cudaStream_t>(stream));
}

// Row collectives: the plan's token split, `outer` batches, rows of row_bytes.
static int rows_collective(const usp_plan* plan, bool reduce, const void* const* src, void* const* dst,
                           int64_t outer, int64_t row_bytes, void* stream) {
  NvtxRange range(reduce ? "usp_reduce_scatter_rows" : "usp_all_gather_rows");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_ptrs(src, plan->world, reduce ? "partial_full_rows" : "local_rows")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(dst), plan->world, reduce ? "local_rows" : "full_rows"))
    return rc;
  if (int rc = device_matches(plan)) return rc;
  if (outer == 0) outer = plan->batch;
  if (row_bytes == 0) row_bytes = static_cast<int64_t>(plan->heads) * plan->head_dim * plan->elem;
  if (outer < 1 || row_bytes < 1) return usp::set_error(USP_ERR_INVALID_ARG, "outer and row_bytes must be positive");
  const int vec = pick_vec(row_bytes);
  if (vec == 0) return usp::set_error(USP_ERR_INVALID_ARG, "row_bytes (%lld) must be even", (long long)row_bytes);
  if (reduce && (row_bytes % plan->elem != 0 || vec < plan->elem))
    return usp::set_error(USP_ERR_INVALID_ARG, "row_bytes (%lld) must be a multiple of the %d-byte element",
                          (long long)row_bytes, plan->elem);
  usp::RowsArgs a;
  memset(&a, 0, sizeof(a));
  a.world = plan->world;
  a.outer = outer;
  a.total_rows = plan->seq_len;
  a.nv = row_bytes / vec;
  for (int r = 0; r < plan->world; ++r) {
    a.tok_start[r] = plan->tok_start[r];
    a.tok_len[r] = plan->tok_len[r];
    a.src[r] = src[r];
    a.dst[r] = dst[r];
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return reduce ? usp::launch_reduce_scatter_rows(a, vec, plan->dtype, s) : usp::launch_all_gather_rows(a, vec, s);
}

int usp_all_gather_rows(const usp_plan* plan, const void* const* local_rows, void* const* full_rows, int64_t outer,
                        int64_t row_bytes, void* stream) {
  return rows_collective(plan, false, local_rows, full_rows, outer, row_bytes, stream);
}

int usp_reduce_scatter_rows(const usp_plan* plan, const void* const* partial_full_rows, void* const* local_rows,
                            int64_t outer, int64_t row_bytes, void* stream) {
  return rows_collective(plan, true, partial_full_rows, local_rows, outer, row_bytes, stream);
}

int usp_ulysses_seq_to_head(const usp_plan* plan, int32_t ntensors, const void* const* in, void* const* out,
                            void* stream) {
  NvtxRange range("usp_ulysses_seq_to_head");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_flat(plan, "usp_ulysses_seq_to_head")) return rc;
  if (ntensors < 1 || ntensors > 3) return usp::set_error(USP_ERR_INVALID_ARG, "ntensors must be 1..3");
  if (int rc = check_ptrs(in, ntensors * plan->world, "in")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(out), ntensors * plan->world, "out")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return seq_head_exchange(plan, 0, ntensors, in, out, static_cast<cudaStream_t>(stream));
}

int usp_ulysses_seq_to_head_kv(const usp_plan* plan, int32_t ntensors, const void* const* in, void* const* out,
                               void* stream) {
  NvtxRange range("usp_ulysses_seq_to_head_kv");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_flat(plan, "usp_ulysses_seq_to_head_kv")) return rc;
  if (ntensors < 1 || ntensors > 3) return usp::set_error(USP_ERR_INVALID_ARG, "ntensors must be 1..3");
  if (int rc = check_ptrs(in, ntensors * plan->world, "in")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(out), ntensors * plan->world, "out")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return seq_head_exchange(plan, 0, ntensors, in, out, static_cast<cudaStream_t>(stream), true);
}

int usp_ulysses_head_to_seq(const usp_plan* plan, int32_t ntensors, const void* const* in, void* const* out,
                            void* stream) {
  NvtxRange range("usp_ulysses_head_to_seq");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_flat(plan, "usp_ulysses_head_to_seq")) return rc;
  if (ntensors < 1 || ntensors > 3) return usp::set_error(USP_ERR_INVALID_ARG, "ntensors must be 1..3");
  if (int rc = check_ptrs(in, ntensors * plan->world, "in")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(out), ntensors * plan->world, "out")) return rc;
  if (int rc = device_matches(plan)) return rc;
  return seq_head_exchange(plan, 1, ntensors, const_cast<const void* const*>(out), const_cast<void* const*>(in),
                           static_cast<cudaStream_t>(stream));
}

static int check_attention_shape(const usp_plan* plan) {
  if (plan->tokens() > (int64_t(1) << 30)) return usp::set_error(USP_ERR_SHAPE, "too many tokens");
  if (plan->dtype == USP_FP32) {
    if (plan->head_dim > 256) return usp::set_error(USP_ERR_UNSUPPORTED, "fp32 attention: head_dim > 256 not built");
  } else if (!usp::attention_tc_supported(plan->dtype, plan->head_dim)) {
    return usp::set_error(USP_ERR_UNSUPPORTED,
                          "16-bit attention needs head_dim a multiple of 16 in [16, 128] (got %d)", plan->head_dim);
  }
  return USP_OK;
}

static int launch_attention(const usp::AttnLaunch& L, cudaStream_t stream) {
  return L.dtype == USP_FP32 ? usp::launch_attention_simt(L, stream) : usp::launch_attention_tc(L, stream);
}

static float resolve_scale(const usp_plan* plan, float scale) {
  return scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(plan->head_dim)));
}

int usp_head_attention(const usp_plan* plan, const void* const* q_heads, const void* const* k_heads,
                       const void* const* v_heads, void* const* o_heads, float scale, void* stream) {
  NvtxRange range("usp_head_attention");
  if (int rc = check_plan(plan)) return rc;
  if (int rc = check_flat(plan, "usp_head_attention")) return rc;
  if (int rc = check_ptrs(q_heads, plan->world, "q_heads")) return rc;
  if (int rc = check_ptrs(k_heads, plan->world, "k_heads")) return rc;
  if (int rc = check_ptrs(v_heads, plan->world, "v_heads")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(o_heads), plan->world, "o_heads")) return rc;
  if (int rc = check_attention_shape(plan)) return rc;
  if (int rc = device_matches(plan)) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t T = plan->tokens(), D = plan->head_dim;
  for (int r = 0; r < plan->world; ++r) {
    usp::AttnLaunch L;
    memset(&L, 0, sizeof(L));
    const int64_t hr = plan->head_len[r];
    const int64_t kr = plan->kv_head_len[r];
    L.in.q = q_heads[r];
    L.in.k = k_heads[r];
    L.in.v = v_heads[r];
    L.in.qv = {D, hr * D, T * hr * D, hr};
    L.in.kvv = {D, kr * D, T * kr * D, kr};
    L.in.kv_group = plan->kv_group;
    L.in.q_head_base = plan->head_start[r];
    L.in.kv_head_base = plan->kv_head_start[r];
    L.out.nseg = 1;
    L.out.prefix = 0;
    L.out.out_heads = static_cast<int32_t>(hr);
    L.out.seg_start[0] = 0;
    L.out.seg_len[0] = T;
    L.out.seg_ptr[0] = o_heads[r];
    L.tokens = static_cast<int32_t>(T);
    L.batch = static_cast<int32_t>(plan->batch);
    L.n_heads = static_cast<int32_t>(hr);
    L.head_dim = static_cast<int32_t>(D);
    L.dtype = plan->dtype;
    L.scale = resolve_scale(plan, scale);
    L.max_ctas = plan->attn_ctas;
    L.kernel = plan->attn_kernel;
    for (int h = 0; h < hr; ++h) L.heads[h] = static_cast<uint16_t>(h);
    if (int rc = launch_attention(L, s)) return rc;
  }
  return USP_OK;
}

// Records a caller's timing event. Under stream capture it is recorded as an
// external event node, so every replay of the graph records it again.
static int record_timing_event(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus status = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &status);
  if (e != cudaSuccess) return usp::cuda_check(e, "cudaStreamIsCapturing");
  const unsigned flags = status == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  return usp::cuda_check(cudaEventRecordWithFlags(ev, s, flags), "cudaEventRecordWithFlags(timing)");
}

// Bytes of one head-major workspace tensor with `heads` heads, 256-byte aligned.
static size_t workspace_tensor_bytes(const usp_plan* plan, int32_t heads) {
  const size_t bytes = static_cast<size_t>(plan->batch) * plan->tokens() * heads * plan->head_dim * plan->elem;
  return (bytes + 255) & ~size_t(255);
}

static size_t workspace_total_bytes(const usp_plan* plan) {
  return workspace_tensor_bytes(plan, plan->heads) + 2 * workspace_tensor_bytes(plan, plan->heads_kv);
}

int usp_ulysses_attention_workspace_size(const usp_plan* plan, int32_t num_chunks, size_t* bytes) {
  if (int rc = check_plan(plan)) return rc;
  if (!bytes) return usp::set_error(USP_ERR_INVALID_ARG, "bytes is NULL");
  if (num_chunks < 1) return usp::set_error(USP_ERR_INVALID_ARG, "num_chunks must be positive");
  *bytes = workspace_total_bytes(plan);
  return USP_OK;
}

// k/v heads packed with chunk window [lo, hi): on every rank, the kv heads whose
// first query head lies in the window, so each kv head is packed exactly once
// and before the first chunk that reads it.
static void select_chunk_kv_heads(usp::PermuteArgs& a, const usp_plan* p, int lo, int hi) {
  a.nsel = 0;
  const int g = p->kv_group;
  for (int r = 0; r < p->head_ranks; ++r) {
    if (lo >= p->head_len[r]) continue;
    const int qa = p->head_start[r] + lo;
    const int qb = p->head_start[r] + (hi < p->head_len[r] ? hi : p->head_len[r]);
    for (int kvh = (qa + g - 1) / g; kvh * g < qb; ++kvh) {
      a.sel_head[a.nsel] = static_cast<uint16_t>(kvh);
      a.sel_rank[a.nsel] = static_cast<uint8_t>(r);
      ++a.nsel;
    }
  }
}

static int ulysses_attention_impl(const usp_plan* plan, const void* const* q, const void* const* k,
                                  const void* const* v, void* const* out, float* lse, float scale, int32_t num_chunks,
                                  void* workspace, size_t workspace_bytes, void* stream);

int usp_ulysses_attention(const usp_plan* plan, const void* const* q, const void* const* k, const void* const* v,
                          void* const* out, float scale, int32_t num_chunks, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return ulysses_attention_impl(plan, q, k, v, out, nullptr, scale, num_chunks, workspace, workspace_bytes, stream);
}

int usp_ulysses_attention_lse(const usp_plan* plan, const void* const* q, const void* const* k, const void* const* v,
                              void* const* out, float* lse, float scale, int32_t num_chunks, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!lse) return usp::set_error(USP_ERR_INVALID_ARG, "lse is NULL");
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return usp::set_error(USP_ERR_ALIGN, "lse must be 4-byte aligned");
  return ulysses_attention_impl(plan, q, k, v, out, lse, scale, num_chunks, workspace, workspace_bytes, stream);
}

static int ulysses_attention_impl(const usp_plan* plan, const void* const* q, const void* const* k,
                                  const void* const* v, void* const* out, float* lse, float scale, int32_t num_chunks,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange range("usp_ulysses_attention");
  if (int rc = check_plan(plan)) return rc;
  // One call's event records, waits and launches are enqueued as a unit.
  std::lock_guard<std::recursive_mutex> guard(plan->lock);
  if (num_chunks < 1) return usp::set_error(USP_ERR_INVALID_ARG, "num_chunks must be positive (got %d)", num_chunks);
  if (int rc = check_ptrs(q, plan->world, "q")) return rc;
  if (int rc = check_ptrs(k, plan->world, "k")) return rc;
  if (int rc = check_ptrs(v, plan->world, "v")) return rc;
  if (int rc = check_ptrs(const_cast<const void* const*>(out), plan->world, "out")) return rc;
  if (!workspace) return usp::set_error(USP_ERR_INVALID_ARG, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return usp::set_error(USP_ERR_ALIGN, "workspace must be 256-byte aligned");
  const size_t need = workspace_total_bytes(plan);
  if (workspace_bytes < need)
    return usp::set_error(USP_ERR_SHAPE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  if (int rc = check_attention_shape(plan)) return rc;
  if (int rc = device_matches(plan)) return rc;

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t T = plan->tokens(), D = plan->head_dim, B = plan->batch, H = plan->heads, HK = plan->heads_kv;
  const bool gqa = plan->kv_group > 1;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* wq = ws;
  void* wk = ws + workspace_tensor_bytes(plan, plan->heads);
  void* wv = static_cast<uint8_t*>(wk) + workspace_tensor_bytes(plan, plan->heads_kv);

  // Head-chunk windows over the largest per-rank head group (rank 0's).
  int32_t nchunks = 0;
  int32_t lo[USP_MAX_HEADS], hi[USP_MAX_HEADS];
  usp_head_chunk_ranges(plan->group_heads, num_chunks, &nchunks, lo, hi);

  // The seq->head exchange writes head-major workspaces [H][B][T'][D] (q) and
  // [Hkv][B][T'][D] (k, v): rank r's head shard is the contiguous block of its
  // heads, so one 4-D view of each workspace covers every rank for the
  // attention kernel. Without grouped-query attention q, k and v move in one
  // launch; with it, q and the k/v pair move in two (different head splits).
  const int64_t unit = D * plan->elem;
  const int vec = pick_vec(unit);
  auto pack_args = [&](usp::PermuteArgs& a, int32_t heads, const int32_t* hstart, int ntensors) {
    memset(&a, 0, sizeof(a));
    a.dir = 0;
    fill_seq_side(a, plan, B);
    a.n_head = plan->head_ranks;
    a.ntensors = ntensors;
    a.heads = heads;
    a.dv = static_cast<int32_t>(unit / vec);
    a.head_layout = 1;
    a.full_tokens = T;
    for (int r = 0; r <= plan->head_ranks; ++r) a.head_start[r] = hstart[r];
  };
  usp::PermuteArgs aq, akv;
  pack_args(aq, static_cast<int32_t>(H), plan->head_start, gqa ? 1 : 3);
  pack_args(akv, static_cast<int32_t>(HK), plan->kv_head_start, 2);
  usp::PermuteArgs& kvargs = gqa ? akv : aq;
  const int t0 = gqa ? 0 : 1;
  for (int r = 0; r < plan->world; ++r) {
    aq.seq_ptr[0][r] = const_cast<void*>(q[r]);
    kvargs.seq_ptr[t0][r] = const_cast<void*>(k[r]);
    kvargs.seq_ptr[t0 + 1][r] = const_cast<void*>(v[r]);
  }
  // Head-side buffers: one per head rank (every rank for the plain block; the
  // Ulysses positions u of the hybrid, where rank (g, u) owns the token block g
  // of head group u's buffer).
  for (int r = 0; r < plan->head_ranks; ++r) {
    const size_t qoff = static_cast<size_t>(plan->head_start[r]) * B * T * D * plan->elem;
    const size_t kvoff = static_cast<size_t>(plan->kv_head_start[r]) * B * T * D * plan->elem;
    aq.head_ptr[0][r] = static_cast<uint8_t*>(wq) + qoff;
    kvargs.head_ptr[t0][r] = static_cast<uint8_t*>(wk) + kvoff;
    kvargs.head_ptr[t0 + 1][r] = static_cast<uint8_t*>(wv) + kvoff;
  }

  usp::AttnLaunch L;
  memset(&L, 0, sizeof(L));
  L.in.q = wq;
  L.in.k = wk;
  L.in.v = wv;
  L.in.qv = {B * T * D, D, T * D, H};
  L.in.kvv = {B * T * D, D, T * D, HK};
  L.in.kv_group = plan->kv_group;
  L.in.q_head_base = 0;
  L.in.kv_head_base = 0;
  L.out.nseg = plan->world;
  L.out.prefix = plan->prefix;
  L.out.out_heads = static_cast<int32_t>(H);
  for (int r = 0; r < plan->world; ++r) {
    L.out.seg_start[r] = plan->tok_start[r];
    L.out.seg_len[r] = plan->tok_len[r];
    L.out.seg_ptr[r] = out[r];
  }
  L.tokens = static_cast<int32_t>(T);
  L.batch = static_cast<int32_t>(B);
  L.head_dim = static_cast<int32_t>(D);
  L.dtype = plan->dtype;
  L.scale = resolve_scale(plan, scale);
  L.max_ctas = plan->attn_ctas;
  L.kernel = plan->attn_kernel;
  L.lse = lse;
  if (plan->ring > 1) {
    // Ring: query group g = key block g = token block of Ulysses group g
    // (block 0 also holds the prefix rows); group g takes the key blocks in
    // ring order g, g-1, ... inside one kernel.
    L.blocks.n_qgroups = L.blocks.n_kvblocks = plan->ring;
    for (int g = 0; g < plan->ring; ++g)
      L.blocks.q_start[g] = L.blocks.kv_start[g] =
          g == 0 ? 0 : static_cast<int32_t>(plan->prefix + plan->tok_start[g * plan->head_ranks]);
    L.blocks.q_start[plan->ring] = L.blocks.kv_start[plan->ring] = static_cast<int32_t>(T);
  }

  const bool overlap = nchunks > 1;
  if (overlap) {
    // Fork: the auxiliary stream packs chunk c+1 while `stream` attends chunk c.
    if (int rc = usp::cuda_check(cudaEventRecord(plan->ev_inputs, s), "cudaEventRecord")) return rc;
    if (int rc = usp::cuda_check(cudaStreamWaitEvent(plan->aux, plan->ev_inputs, 0), "cudaStreamWaitEvent")) return rc;
  }
  const cudaStream_t ps = overlap ? plan->aux : s;
  for (int c = 0; c < nchunks; ++c) {
    char range_name[64];
    snprintf(range_name, sizeof(range_name), "usp chunk %d/%d: pack + attention", c + 1, nchunks);
    NvtxRange chunk_range(range_name);
    select_chunk_heads(aq, plan, lo[c], hi[c]);
    if (int rc = launch_pack(plan, aq, vec, unit, ps)) return rc;
    if (gqa) {
      select_chunk_kv_heads(akv, plan, lo[c], hi[c]);
      if (int rc = launch_pack(plan, akv, vec, unit, ps)) return rc;
    }
    if (overlap) {
      if (int rc = usp::cuda_check(cudaEventRecord(plan->ev_chunk[c], plan->aux), "cudaEventRecord")) return rc;
      if (int rc = usp::cuda_check(cudaStreamWaitEvent(s, plan->ev_chunk[c], 0), "cudaStreamWaitEvent")) return rc;
    }
    L.n_heads = aq.nsel;
    for (int i = 0; i < aq.nsel; ++i) L.heads[i] = aq.sel_head[i];
    if (c == 0 && plan->t_start)
      if (int rc = record_timing_event(plan->t_start, s)) return rc;
    if (int rc = launch_attention(L, s)) return rc;
  }
  if (plan->t_stop)
    if (int rc = record_timing_event(plan->t_stop, s)) return rc;
  return USP_OK;
}

struct usp_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int device = 0;
};

int usp_ulysses_attention_graph_create(usp_graph** out, const usp_plan* plan, const void* const* q,
                                       const void* const* k, const void* const* v, void* const* o, float scale,
                                       int32_t num_chunks, void* workspace, size_t workspace_bytes) {
  if (!out) return usp::set_error(USP_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (int rc = check_plan(plan)) return rc;
  if (int rc = device_matches(plan)) return rc;
  NvtxRange range("usp_ulysses_attention_graph_create");
  // No other call may enqueue on the plan's auxiliary stream while the capture
  // has pulled it in.
  std::lock_guard<std::recursive_mutex> guard(plan->lock);
  cudaStream_t cap = nullptr;
  if (int rc = usp::cuda_check(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking), "cudaStreamCreate")) return rc;
  int rc = usp::cuda_check(cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal), "cudaStreamBeginCapture");
  cudaGraph_t graph = nullptr;
  if (rc == USP_OK) {
    // The call validates every argument and records only stream-ordered work.
    const int call_rc = usp_ulysses_attention(plan, q, k, v, o, scale, num_chunks, workspace, workspace_bytes, cap);
    const std::string call_msg = g_last_error;
    const cudaError_t end = cudaStreamEndCapture(cap, &graph);
    if (call_rc != USP_OK) {
      rc = call_rc;
      g_last_error = call_msg;
    } else {
      rc = usp::cuda_check(end, "cudaStreamEndCapture");
    }
  }
  cudaStreamDestroy(cap);
  if (rc != USP_OK) {
    if (graph) cudaGraphDestroy(graph);
    return rc;
  }
  usp_graph* g = new usp_graph();
  g->graph = graph;
  g->device = plan->device;
  if ((rc = usp::cuda_check(cudaGraphInstantiate(&g->exec, graph, 0), "cudaGraphInstantiate")) != USP_OK) {
    usp_graph_destroy(g);
    return rc;
  }
  *out = g;
  return USP_OK;
}

int usp_graph_launch(usp_graph* graph, void* stream) {
  if (!graph) return usp::set_error(USP_ERR_INVALID_ARG, "graph is NULL");
  int dev = -1;
  if (int rc = usp::cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  if (dev != graph->device)
    return usp::set_error(USP_ERR_INVALID_ARG, "graph was captured on device %d but device %d is current",
                          graph->device, dev);
  return usp::cuda_check(cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)), "cudaGraphLaunch");
}

int usp_graph_destroy(usp_graph* graph) {
  if (!graph) return USP_OK;
  if (graph->exec) cudaGraphExecDestroy(graph->exec);
  if (graph->graph) cudaGraphDestroy(graph->graph);
  delete graph;
  return USP_OK;
}

int usp_plan_set_pack_mode(usp_plan* plan, int32_t mode) {
  if (int rc = check_plan(plan)) return rc;
  if (mode != USP_PACK_VECTOR && mode != USP_PACK_TMA)
    return usp::set_error(USP_ERR_INVALID_ARG, "pack mode must be USP_PACK_VECTOR or USP_PACK_TMA (got %d)", mode);
  plan->pack_mode = mode;
  return USP_OK;
}

int usp_plan_set_attention_ctas(usp_plan* plan, int32_t max_ctas) {
  if (int rc = check_plan(plan)) return rc;
  if (max_ctas < 0) return usp::set_error(USP_ERR_INVALID_ARG, "attention CTA cap must be >= 0 (got %d)", max_ctas);
  plan->attn_ctas = max_ctas;
  return USP_OK;
}

int usp_plan_set_attention_kernel(usp_plan* plan, int32_t kernel) {
  if (int rc = check_plan(plan)) return rc;
  if (kernel != USP_ATTN_AUTO && kernel != USP_ATTN_ONE_TILE && kernel != USP_ATTN_TWO_TILE &&
      kernel != USP_ATTN_TWO_CTA)
    return usp::set_error(USP_ERR_INVALID_ARG, "unknown attention kernel %d", kernel);
  if (kernel == USP_ATTN_TWO_TILE && !usp::attention_pp_supported(plan->dtype, plan->head_dim, kernel))
    return usp::set_error(USP_ERR_UNSUPPORTED, "the two-query-tile kernel takes 16-bit inputs with head_dim a "
                          "multiple of 16 in [64, 128] (got dtype %d, head_dim %d)", plan->dtype, plan->head_dim);
  if (kernel == USP_ATTN_TWO_CTA && !usp::attention_pp_supported(plan->dtype, plan->head_dim, kernel))
    return usp::set_error(USP_ERR_UNSUPPORTED, "the two-CTA kernel takes 16-bit inputs with head_dim 64 or 80 "
                          "(got dtype %d, head_dim %d)", plan->dtype, plan->head_dim);
  std::lock_guard<std::recursive_mutex> guard(plan->lock);
  plan->attn_kernel = kernel;
  return USP_OK;
}

int usp_plan_set_timing_events(usp_plan* plan, void* start, void* stop) {
  if (int rc = check_plan(plan)) return rc;
  std::lock_guard<std::recursive_mutex> guard(plan->lock);
  if ((start == nullptr) != (stop == nullptr))
    return usp::set_error(USP_ERR_INVALID_ARG, "set both timing events or neither");
  plan->t_start = static_cast<cudaEvent_t>(start);
  plan->t_stop = static_cast<cudaEvent_t>(stop);
  return USP_OK;
}

uint64_t usp_kernel_launches(void) { return usp::g_launches.load(std::memory_order_relaxed); }

int usp_device_status(uint32_t* code, int32_t reset) {
  if (!code) return usp::set_error(USP_ERR_INVALID_ARG, "code is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return usp::cuda_check(e, "cudaDeviceSynchronize");
  if (int rc = usp::read_attention_error(code, reset != 0)) return rc;
  uint32_t pack_code = 0, pp_code = 0;
  if (int rc = usp::read_pack_error(&pack_code, reset != 0)) return rc;
  if (int rc = usp::read_pp_error(&pp_code, reset != 0)) return rc;
  if (*code == 0) *code = pack_code;
  if (*code == 0) *code = pp_code;
  if (*code != 0) {
    usp::set_error(USP_ERR_TIMEOUT, "a device-side wait ran out (site %u)", *code);
    return USP_ERR_TIMEOUT;
  }
  // Bounds-checking builds record the first out-of-range access per kernel file.
  int (*const readers[])(uint32_t*, bool) = {usp::read_permute_bounds, usp::read_rows_bounds,
                                             usp::read_pack_bounds, usp::read_attention_bounds,
                                             usp::read_simt_bounds, usp::read_pp_bounds};
  for (auto read : readers) {
    uint32_t site = 0;
    if (int rc = read(&site, reset != 0)) return rc;
    if (*code == 0) *code = site;
  }
  if (*code != 0) {
    usp::set_error(USP_ERR_BOUNDS, "an out-of-range offset was skipped (site %u)", *code);
    return USP_ERR_BOUNDS;
  }
  return USP_OK;
}

int usp_debug_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 2000000) return usp::set_error(USP_ERR_INVALID_ARG, "limit_us must be in [1, 2e6]");
  return usp::launch_wait_timeout_probe(limit_us, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// Helpers shared with the rank-local (multi-process) entry points in dist.cpp.
namespace usp {

int plan_vec_bytes(const usp_plan* plan) { return pick_vec(static_cast<int64_t>(plan->head_dim) * plan->elem); }

int plan_launch_pack(const usp_plan* plan, const PermuteArgs& a, cudaStream_t stream) {
  const int64_t unit = static_cast<int64_t>(plan->head_dim) * plan->elem;
  return launch_pack(plan, a, pick_vec(unit), unit, stream);
}

int plan_check_ptr(const void* p, const char* what) { return check_ptr(p, what); }

int plan_check_device(const usp_plan* plan) { return device_matches(plan); }

int plan_check_attention(const usp_plan* plan) { return check_attention_shape(plan); }

int plan_launch_attention(const AttnLaunch& L, cudaStream_t stream) { return launch_attention(L, stream); }

float plan_scale(const usp_plan* plan, float scale) { return resolve_scale(plan, scale); }

}  // namespace usp
