// Ragged row permutation between sequence shards and head shards.
//
// Every layout step of the Ulysses block moves whole head units (D elements)
// between a buffer that holds complete token rows (the "sequence side") and a
// buffer that holds a contiguous head range for every token (the "head
// side"):
//   seq->head exchange  ("h3_blackwell_runtime/distributed.py", seq_to_heads)
//   head->seq exchange  (heads_to_seq)
//   head slice / gather (API page)
// (scatter / gather of the sequence, whose rows are contiguous on both sides,
// run as a segmented copy in rows.cu.) The kernel walks the sequence-side rows, so that side is read or written in
// full contiguous rows; each head unit is a contiguous run of D*elem bytes on
// the head side. A warp moves one segment of a row at a time (32 lanes x 4
// vectors of 2..16 bytes), all loads of a segment issued before its stores.
#include <cstdio>

#include "device_common.cuh"
#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {
__device__ uint32_t g_permute_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;
constexpr int kUnitBatches = 4;  // unrolled batches of kUnroll vectors per lane in one work unit

template <typename V>
__global__ void __launch_bounds__(kThreads, 4) permute_kernel(const __grid_constant__ PermuteArgs a) {
  __shared__ int32_t s_unit[USP_MAX_HEADS];    // head unit index on the sequence side
  __shared__ int32_t s_rank[USP_MAX_HEADS];    // head-side buffer
  __shared__ int32_t s_local[USP_MAX_HEADS];   // unit index inside that buffer
  __shared__ int32_t s_count[USP_MAX_HEADS];   // units held by that buffer
  for (int i = threadIdx.x; i < a.nsel; i += blockDim.x) {
    const int h = a.sel_head[i];
    const int r = a.sel_rank[i];
    s_unit[i] = h - a.seq_unit_base;
    s_rank[i] = r;
    s_local[i] = h - a.head_start[r];
    s_count[i] = head_units(a, r);
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const int64_t total_rows = a.seq_rows[a.n_seq];
  const int nvec = a.nsel * a.dv;
  // Work is dealt out in segments of a row (kUnitBatches unrolled batches of
  // 32 * kUnroll vectors), one per warp; the grid normally covers every
  // segment, and the loop only takes over beyond the largest grid.
  constexpr int kBatch = 32 * kUnroll;
  constexpr int kSeg = kBatch * kUnitBatches;
  const int nseg = (nvec + kSeg - 1) / kSeg;
  const int64_t total_units = total_rows * nseg;

  for (int64_t unit = warp; unit < total_units; unit += nwarps) {
    const int64_t row = unit / nseg;
    const int seg = static_cast<int>(unit - row * nseg);
    int s = 0;
    while (a.seq_rows[s + 1] <= row) ++s;
    const int64_t rr = row - a.seq_rows[s];
    const int64_t rows_per_b = a.prefix + a.tok_len[s];
    const int64_t b = rr / rows_per_b;
    const int64_t tl = rr - b * rows_per_b;
    // Replicated prefix rows: read once (from buffer 0) on the way to the head
    // side, written to every sequence-side buffer on the way back.
    if (a.dir == 0 && tl < a.prefix && s != 0) continue;
    const int64_t t = (tl < a.prefix) ? tl : a.prefix + a.tok_start[s] + (tl - a.prefix);
    const int64_t seq_base = rr * a.heads * a.dv;

    const int j_end = min(nvec, (seg + 1) * kSeg);
    for (int j0 = seg * kSeg; j0 < j_end; j0 += kBatch) {
      int64_t soff[kUnroll], hoff[kUnroll];
      int hr[kUnroll];
      bool ok[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = j0 + u * 32 + lane;
        ok[u] = j < j_end;
        const int k = ok[u] ? j / a.dv : 0;
        const int d = j - k * a.dv;
        const int64_t hl = s_local[k];
        const int64_t cr = s_count[k];
        hr[u] = s_rank[k];
        soff[u] = seq_base + static_cast<int64_t>(s_unit[k]) * a.dv + d;
        hoff[u] = (a.head_layout == 0) ? ((b * a.full_tokens + t) * cr + hl) * a.dv + d
                                       : ((hl * a.outer + b) * a.full_tokens + t) * a.dv + d;
      }
      for (int ti = 0; ti < a.ntensors; ++ti) {
        V val[kUnroll];
        if (a.dir == 0) {
          const V* src = static_cast<const V*>(a.seq_ptr[ti][s]);
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (ok[u] && in_bounds(soff[u], 1, a.seq_ext[s], 1, &g_permute_bounds)) val[u] = __ldcs(src + soff[u]);
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (ok[u] && in_bounds(hoff[u], 1, a.head_ext[hr[u]], 2, &g_permute_bounds))
              __stcs(static_cast<V*>(a.head_ptr[ti][hr[u]]) + hoff[u], val[u]);
        } else {
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (ok[u] && in_bounds(hoff[u], 1, a.head_ext[hr[u]], 3, &g_permute_bounds))
              val[u] = __ldcs(static_cast<const V*>(a.head_ptr[ti][hr[u]]) + hoff[u]);
          V* dst = static_cast<V*>(a.seq_ptr[ti][s]);
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (ok[u] && in_bounds(soff[u], 1, a.seq_ext[s], 4, &g_permute_bounds)) __stcs(dst + soff[u], val[u]);
        }
      }
    }
  }
}

}  // namespace

int sm_count() {
  int dev = 0, count = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    count = 148;
  return count;
}

int launch_permute(const PermuteArgs& args, int vec_bytes, cudaStream_t stream) {
  PermuteArgs a = args;
  for (int s = 0; s < a.n_seq; ++s) a.seq_ext[s] = (a.seq_rows[s + 1] - a.seq_rows[s]) * a.heads * a.dv;
  for (int r = 0; r < a.n_head; ++r)
    a.head_ext[r] = a.outer * a.full_tokens * head_units(a, r) * a.dv;
  const int64_t rows = a.seq_rows[a.n_seq];
  if (rows == 0 || a.nsel == 0) return USP_OK;
  // Work units of 4 batches (up to 512 vectors of a row), one CTA of 8 warps
  // per 8 units and no grid-stride loop: measured on the reshard workload,
  // this beat one resident wave of CTAs looping over 1-batch units by 4-9%
  // (the CTAs' launch and drain overlap instead of each CTA's next loads
  // waiting behind its stores).
  a.unit_batches = kUnitBatches;
  const int64_t nvec = static_cast<int64_t>(a.nsel) * a.dv;
  const int64_t seg = 32 * kUnroll * a.unit_batches;
  const int64_t warps_needed = rows * ((nvec + seg - 1) / seg);
  int64_t blocks = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
  if (blocks > 0x7fffffff) blocks = 0x7fffffff;  // then the kernel's unit loop takes the rest
  dim3 grid(static_cast<unsigned>(blocks)), block(kThreads);
  switch (vec_bytes) {
    case 16: permute_kernel<uint4><<<grid, block, 0, stream>>>(a); break;
    case 8: permute_kernel<uint2><<<grid, block, 0, stream>>>(a); break;
    case 4: permute_kernel<uint32_t><<<grid, block, 0, stream>>>(a); break;
    case 2: permute_kernel<uint16_t><<<grid, block, 0, stream>>>(a); break;
    default: return set_error(USP_ERR_INVALID_ARG, "internal: bad vector width %d", vec_bytes);
  }
  count_launch();
  return cuda_check(cudaGetLastError(), "permute kernel launch");
}

int read_permute_bounds(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_permute_bounds, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read permute bounds word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_permute_bounds, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset permute bounds word");
  }
  return USP_OK;
}

}  // namespace usp
