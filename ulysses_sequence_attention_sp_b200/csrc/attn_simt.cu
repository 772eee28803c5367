// Non-causal softmax attention in fp32 on the CUDA cores.
//
// Same operation and output routing as the tcgen05 kernel (API page
// "mstar.model.components.distributed.sequence_parallel", ulysses_attention /
// run_attention), for fp32 inputs, where the tensor-core fp32 paths (tf32)
// would not hold fp32 accuracy. Four threads share one query row; each holds a
// quarter of the head dimension of q and of the accumulator. Keys and values
// are staged through shared memory 32 rows at a time; the online softmax runs
// in the log2 domain with exact exp2f.
#include <cmath>

#include "device_common.cuh"
#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_simt_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

namespace {

constexpr int kTPR = 4;                  // threads per query row
constexpr int kThreads = 128;
constexpr int kRows = kThreads / kTPR;   // query rows per CTA
constexpr int kKT = 32;                  // keys per smem tile

struct SimtBlocks {
  int32_t nq, nk;
  int32_t q_start[USP_MAX_WORLD + 1];
  int32_t q_tile_prefix[USP_MAX_WORLD + 1];
  int32_t kv_start[USP_MAX_WORLD + 1];
};

template <int DPT>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(const __grid_constant__ AttnLaunch L,
                                                             const __grid_constant__ SimtBlocks B, float scale_log2) {
  extern __shared__ float sh[];
  const int D = L.head_dim;
  const int DP = DPT * kTPR;  // padded head dim
  float* sk = sh;
  float* sv = sh + kKT * DP;

  const int hi = blockIdx.y / L.batch;
  const int b = blockIdx.y - hi * L.batch;
  const int hm = L.heads[hi];
  const int T = L.tokens;
  const int sub = threadIdx.x % kTPR;
  // query group of this CTA; its rows are [q_start[g], q_start[g+1])
  int g = 0;
  while (g + 1 < B.nq && static_cast<int>(blockIdx.x) >= B.q_tile_prefix[g + 1]) ++g;
  const int row = B.q_start[g] + (static_cast<int>(blockIdx.x) - B.q_tile_prefix[g]) * kRows + threadIdx.x / kTPR;
  const bool row_ok = row < B.q_start[g + 1];

  const int hk = (L.in.q_head_base + hm) / L.in.kv_group - L.in.kv_head_base;  // kv head of this query head
  const float* qb = static_cast<const float*>(L.in.q) + hm * L.in.qv.stride_head + b * L.in.qv.stride_batch;
  const float* kb = static_cast<const float*>(L.in.k) + hk * L.in.kvv.stride_head + b * L.in.kvv.stride_batch;
  const float* vb = static_cast<const float*>(L.in.v) + hk * L.in.kvv.stride_head + b * L.in.kvv.stride_batch;

  float q[DPT], acc[DPT];
#pragma unroll
  for (int i = 0; i < DPT; ++i) {
    const int d = sub * DPT + i;
    q[i] = (row_ok && d < D) ? qb[static_cast<int64_t>(row) * L.in.qv.stride_token + d] * scale_log2 : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  // key blocks in ring order g, g-1, ... (mod nk); each in smem tiles of kKT keys
  int blk = g % B.nk;
  for (int step = 0; step < B.nk; ++step, blk = blk == 0 ? B.nk - 1 : blk - 1)
  for (int k0 = B.kv_start[blk]; k0 < B.kv_start[blk + 1]; k0 += kKT) {
    const int kend = B.kv_start[blk + 1];
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKT * DP; idx += kThreads) {
      const int r = idx / DP, d = idx - r * DP;
      const bool ok = (k0 + r < kend) && d < D;
      const int64_t off = static_cast<int64_t>(k0 + r) * L.in.kvv.stride_token + d;
      sk[idx] = ok ? kb[off] : 0.f;
      sv[idx] = ok ? vb[off] : 0.f;
    }
    __syncthreads();
    const int nk = min(kKT, kend - k0);
    float s[kKT];
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < kKT; ++r) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < DPT; ++i) dot = fmaf(q[i], sk[r * DP + sub * DPT + i], dot);
#pragma unroll
      for (int o = 1; o < kTPR; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      s[r] = (r < nk) ? dot : -INFINITY;
      mx = fmaxf(mx, s[r]);
    }
    const float m_new = fmaxf(m, mx);
    const float alpha = exp2f(m - m_new);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < DPT; ++i) acc[i] *= alpha;
#pragma unroll
    for (int r = 0; r < kKT; ++r) {
      const float pr = exp2f(s[r] - m_new);
      l += pr;
#pragma unroll
      for (int i = 0; i < DPT; ++i) acc[i] = fmaf(pr, sv[r * DP + sub * DPT + i], acc[i]);
    }
    m = m_new;
  }
  if (!row_ok) return;
  if (L.lse != nullptr && sub == 0) {  // sum_j exp(scale s_j) = 2^m * l
    const int64_t li = (static_cast<int64_t>(hm) * L.batch + b) * T + row;
    if (in_bounds(li, 1, static_cast<int64_t>(L.in.qv.head_extent) * L.batch * T, 42, &g_simt_bounds))
      L.lse[li] = (m + log2f(l)) * 0.69314718055994531f;
  }

  const AttnOut& out = L.out;
  int seg_lo, seg_hi;
  int64_t row_in_seg;
  if (row < out.prefix) {
    seg_lo = 0;
    seg_hi = out.nseg;
    row_in_seg = row;
  } else {
    const int64_t tok = row - out.prefix;
    int s = 0;
    while (s + 1 < out.nseg && tok >= out.seg_start[s + 1]) ++s;
    seg_lo = s;
    seg_hi = s + 1;
    row_in_seg = out.prefix + tok - out.seg_start[s];
  }
  const float inv_l = 1.f / l;
  for (int s = seg_lo; s < seg_hi; ++s) {
    const int64_t rows_s = out.prefix + out.seg_len[s];
    const int64_t base = ((b * rows_s + row_in_seg) * out.out_heads + hm - out.head_base) * D;
    float* dst = static_cast<float*>(out.seg_ptr[s]) + base;
    const int64_t ext = static_cast<int64_t>(L.batch) * rows_s * out.out_heads * D;  // bounds-checking builds
#pragma unroll
    for (int i = 0; i < DPT; ++i) {
      const int d = sub * DPT + i;
      if (d < D && in_bounds(base + d, 1, ext, 41, &g_simt_bounds)) dst[d] = acc[i] * inv_l;
    }
  }
}

template <int DPT>
int launch_dpt(const AttnLaunch& L, cudaStream_t stream) {
  const size_t smem = 2 * kKT * DPT * kTPR * sizeof(float);
  if (smem > 48 * 1024)
    if (int rc = ensure_smem_limit(reinterpret_cast<const void*>(attn_simt_kernel<DPT>), smem,
                                   "cudaFuncSetAttribute(simt smem)"))
      return rc;
  const float scale_log2 = static_cast<float>(static_cast<double>(L.scale) * 1.4426950408889634);
  SimtBlocks B;
  const int kv_tokens = L.kv_tokens > 0 ? L.kv_tokens : L.tokens;
  if (!fill_blocks(L, kv_tokens, kRows, B.nq, B.nk, B.q_start, B.q_tile_prefix, B.kv_start))
    return set_error(USP_ERR_INVALID_ARG, "internal: bad query-group or key-block table");
  dim3 grid(B.q_tile_prefix[B.nq], L.batch * L.n_heads);
  attn_simt_kernel<DPT><<<grid, kThreads, smem, stream>>>(L, B, scale_log2);
  count_launch();
  return cuda_check(cudaGetLastError(), "attention (fp32) launch");
}

}  // namespace

int launch_attention_simt(const AttnLaunch& L, cudaStream_t stream) {
  if (L.n_heads == 0 || L.batch == 0 || L.tokens == 0) return USP_OK;
  if (L.dtype != USP_FP32) return set_error(USP_ERR_UNSUPPORTED, "fp32 attention kernel called with a 16-bit type");
  const int D = L.head_dim;
  if (D <= 16) return launch_dpt<4>(L, stream);
  if (D <= 32) return launch_dpt<8>(L, stream);
  if (D <= 64) return launch_dpt<16>(L, stream);
  if (D <= 128) return launch_dpt<32>(L, stream);
  if (D <= 256) return launch_dpt<64>(L, stream);
  return set_error(USP_ERR_UNSUPPORTED, "head_dim %d > 256 is not built", D);
}

int read_simt_bounds(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_simt_bounds, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read fp32 attention bounds word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_simt_bounds, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset fp32 attention bounds word");
  }
  return USP_OK;
}

}  // namespace usp
