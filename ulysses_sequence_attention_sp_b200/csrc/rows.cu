// Ragged row collectives of the sequence-parallel context over virtual ranks
// ("h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
// transport", SequenceParallelContext.all_gather_rows / reduce_scatter_rows),
// and the scatter / gather of the sequence (API page, scatter_sequence /
// gather_sequence) as a segmented copy of the same design.
//
// Both are HBM-bound. Work is cut into tiles of kThreads * kU vectors inside
// one contiguous (rank, batch) segment, so a tile's addresses need no per-row
// index arithmetic: a segment of rank r is the T_r rows of one batch element,
// which are contiguous both in r's local buffer [B][T_r][row] and in a full
// buffer [B][T][row] (at row offset tok_start[r]). The grid has one CTA per
// tile: measured on the reshard workload, that beat one resident wave of CTAs
// looping over the tiles by 12-14% (CTAs launch and drain overlapped, instead
// of each CTA's next loads waiting behind its own stores).
//
// all_gather_rows: each local vector is read once and stored into all P full
// buffers (read S, write P*S).
// reduce_scatter_rows: output vector j of rank r is the sum over source ranks
// i = 0..P-1, in that order, of partial i's vector at the same place of the
// full layout; fp32 accumulation, one rounding to the storage type (read P*S,
// write S). Loads of kR ranks are issued before they are added, so each
// thread keeps kR * kU vectors in flight.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "bounds_check.cuh"
#include "usp_internal.h"

namespace usp {

__device__ uint32_t g_rows_bounds;  // bounds-checking builds: first out-of-range site, 0 if none

namespace {

constexpr int kThreads = 256;

struct TileMap {
  int r;
  int64_t b;
  int64_t k;  // tile index inside the (r, b) segment
};

__device__ __forceinline__ TileMap map_tile(const RowsArgs& a, int64_t tile) {
  TileMap m;
  int r = 0;
  while (r + 1 < a.world && tile >= a.tile_prefix[r + 1]) ++r;
  const int64_t q = tile - a.tile_prefix[r];
  m.r = r;
  m.b = q / a.seg_tiles[r];
  m.k = q - m.b * a.seg_tiles[r];
  return m;
}

template <typename V, int kU>
__global__ void __launch_bounds__(kThreads) all_gather_rows_kernel(const __grid_constant__ RowsArgs a) {
  constexpr int64_t kTile = static_cast<int64_t>(kThreads) * kU;
  for (int64_t tile = blockIdx.x; tile < a.tile_prefix[a.world]; tile += gridDim.x) {
    const TileMap m = map_tile(a, tile);
    const int64_t seg_len = a.tok_len[m.r] * a.nv;
    const V* src = static_cast<const V*>(a.src[m.r]) + m.b * seg_len;
    const int64_t doff = (m.b * a.total_rows + a.tok_start[m.r]) * a.nv;
    const int64_t base = m.k * kTile + threadIdx.x;
    V val[kU];
    bool ok[kU];
    const int64_t src_ext = a.outer * a.tok_len[m.r] * a.nv;  // bounds-checking builds only
    const int64_t dst_ext = a.outer * a.total_rows * a.nv;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t j = base + u * kThreads;
      ok[u] = j < seg_len;
      if (ok[u] && in_bounds(m.b * seg_len + j, 1, src_ext, 11, &g_rows_bounds)) val[u] = __ldcs(src + j);
    }
    for (int d = 0; d < a.world; ++d) {
      V* dst = static_cast<V*>(a.dst[d]) + doff;
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (ok[u] && in_bounds(doff + base + u * kThreads, 1, dst_ext, 12, &g_rows_bounds))
          __stcs(dst + base + u * kThreads, val[u]);
    }
  }
}

// scatter_sequence / gather_sequence as a segmented copy: tiles of
// kThreads * kU 16-byte vectors inside one contiguous (segment kind, batch)
// run, all loads of a tile issued before its stores.
template <int kU>
__global__ void __launch_bounds__(kThreads) copy_rows_kernel(const __grid_constant__ CopyArgs a) {
  constexpr int64_t kTile = static_cast<int64_t>(kThreads) * kU;
  const int64_t full_ext = a.outer * a.full_rows * a.nv;  // bounds-checking builds only
  for (int64_t tile = blockIdx.x; tile < a.tile_prefix[a.nkinds]; tile += gridDim.x) {
    int s = 0;
    while (s + 1 < a.nkinds && tile >= a.tile_prefix[s + 1]) ++s;
    const int64_t q = tile - a.tile_prefix[s];
    const int64_t b = q / a.seg_tiles[s];
    const int64_t base = (q - b * a.seg_tiles[s]) * kTile + threadIdx.x;
    const int64_t seg_len = a.rows[s] * a.nv;
    const int64_t soff = (b * a.shard_rows[s] + a.srow0[s]) * a.nv;
    const int64_t foff = (b * a.full_rows + a.frow0[s]) * a.nv;
    const int64_t shard_ext = a.outer * a.shard_rows[s] * a.nv;
    uint4* shard = static_cast<uint4*>(a.shards[a.shard[s]]);
    uint4* full = static_cast<uint4*>(a.full);
    const uint4* src = a.to_shards ? full + foff : shard + soff;
    uint4* dst = a.to_shards ? shard + soff : full + foff;
    const int64_t src_off = a.to_shards ? foff : soff, dst_off = a.to_shards ? soff : foff;
    const int64_t src_ext = a.to_shards ? full_ext : shard_ext, dst_ext = a.to_shards ? shard_ext : full_ext;
    uint4 val[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t j = base + u * kThreads;
      if (j < seg_len && in_bounds(src_off + j, 1, src_ext, 15, &g_rows_bounds)) val[u] = __ldcs(src + j);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t j = base + u * kThreads;
      if (j < seg_len && in_bounds(dst_off + j, 1, dst_ext, 16, &g_rows_bounds)) __stcs(dst + j, val[u]);
    }
  }
}

template <typename E>
__device__ __forceinline__ float to_f32(E x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

template <typename E>
__device__ __forceinline__ E from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <>
__device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

template <typename V, typename E>
union Pack {
  V v;
  E e[sizeof(V) / sizeof(E)];
};

template <typename V, typename E, int kU, int kR>
__global__ void __launch_bounds__(kThreads) reduce_scatter_rows_kernel(const __grid_constant__ RowsArgs a) {
  constexpr int kE = sizeof(V) / sizeof(E);
  constexpr int64_t kTile = static_cast<int64_t>(kThreads) * kU;
  for (int64_t tile = blockIdx.x; tile < a.tile_prefix[a.world]; tile += gridDim.x) {
    const TileMap m = map_tile(a, tile);
    const int64_t seg_len = a.tok_len[m.r] * a.nv;
    const int64_t soff = (m.b * a.total_rows + a.tok_start[m.r]) * a.nv;
    const int64_t base = m.k * kTile + threadIdx.x;
    bool ok[kU];
    float acc[kU][kE];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      ok[u] = base + u * kThreads < seg_len;
#pragma unroll
      for (int e = 0; e < kE; ++e) acc[u][e] = -0.0f;  // -0 + x == x for every x, signed zeros included
    }
    for (int i0 = 0; i0 < a.world; i0 += kR) {
      Pack<V, E> x[kR][kU];
#pragma unroll
      for (int q = 0; q < kR; ++q) {
        if (i0 + q < a.world) {
          const V* src = static_cast<const V*>(a.src[i0 + q]) + soff;
#pragma unroll
          for (int u = 0; u < kU; ++u)
            if (ok[u] && in_bounds(soff + base + u * kThreads, 1, a.outer * a.total_rows * a.nv, 13, &g_rows_bounds))
              x[q][u].v = __ldcs(src + base + u * kThreads);
        }
      }
#pragma unroll
      for (int q = 0; q < kR; ++q) {
        if (i0 + q < a.world) {
#pragma unroll
          for (int u = 0; u < kU; ++u)
#pragma unroll
            for (int e = 0; e < kE; ++e) acc[u][e] += to_f32<E>(x[q][u].e[e]);
        }
      }
    }
    V* dst = static_cast<V*>(a.dst[m.r]) + m.b * seg_len;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (!ok[u] ||
          !in_bounds(m.b * seg_len + base + u * kThreads, 1, a.outer * a.tok_len[m.r] * a.nv, 14, &g_rows_bounds))
        continue;
      Pack<V, E> o;
#pragma unroll
      for (int e = 0; e < kE; ++e) o.e[e] = from_f32<E>(acc[u][e]);
      __stcs(dst + base + u * kThreads, o.v);
    }
  }
}

// Tiles per (rank, batch) segment and their prefix sums over ranks.
int64_t fill_tiles(RowsArgs& a, int64_t tile_vectors) {
  a.tile_prefix[0] = 0;
  for (int r = 0; r < a.world; ++r) {
    a.seg_tiles[r] = (a.tok_len[r] * a.nv + tile_vectors - 1) / tile_vectors;
    a.tile_prefix[r + 1] = a.tile_prefix[r] + a.outer * a.seg_tiles[r];
  }
  return a.tile_prefix[a.world];
}

// One CTA per tile (the kernels' tile loops take the rest beyond the largest grid).
unsigned grid_for(int64_t tiles) { return static_cast<unsigned>(tiles < 0x7fffffff ? tiles : 0x7fffffff); }

template <typename V>
int gather_v(RowsArgs a, cudaStream_t s) {
  constexpr int kU = 4;
  const int64_t tiles = fill_tiles(a, static_cast<int64_t>(kThreads) * kU);
  if (tiles == 0) return USP_OK;
  auto* k = all_gather_rows_kernel<V, kU>;
  k<<<grid_for(tiles), kThreads, 0, s>>>(a);
  count_launch();
  return cuda_check(cudaGetLastError(), "all_gather_rows launch");
}

template <typename V, typename E>
int reduce_v(RowsArgs a, cudaStream_t s) {
  constexpr int kU = 2, kR = 4;
  const int64_t tiles = fill_tiles(a, static_cast<int64_t>(kThreads) * kU);
  if (tiles == 0) return USP_OK;
  auto* k = reduce_scatter_rows_kernel<V, E, kU, kR>;
  k<<<grid_for(tiles), kThreads, 0, s>>>(a);
  count_launch();
  return cuda_check(cudaGetLastError(), "reduce_scatter_rows launch");
}

template <typename E>
int reduce_e(const RowsArgs& a, int vec_bytes, cudaStream_t s) {
  switch (vec_bytes) {
    case 16: return reduce_v<uint4, E>(a, s);
    case 8: return reduce_v<uint2, E>(a, s);
    case 4:
      if constexpr (sizeof(E) <= 4) return reduce_v<uint32_t, E>(a, s);
      break;
    case 2:
      if constexpr (sizeof(E) <= 2) return reduce_v<uint16_t, E>(a, s);
      break;
  }
  return set_error(USP_ERR_INVALID_ARG, "internal: vector width %d for a %d-byte element", vec_bytes,
                   static_cast<int>(sizeof(E)));
}

}  // namespace

int launch_all_gather_rows(const RowsArgs& a, int vec_bytes, cudaStream_t s) {
  switch (vec_bytes) {
    case 16: return gather_v<uint4>(a, s);
    case 8: return gather_v<uint2>(a, s);
    case 4: return gather_v<uint32_t>(a, s);
    case 2: return gather_v<uint16_t>(a, s);
    default: return set_error(USP_ERR_INVALID_ARG, "internal: bad vector width %d", vec_bytes);
  }
}

int launch_copy_rows(const CopyArgs& args, cudaStream_t s) {
  CopyArgs a = args;
  constexpr int kU = 8;  // 32 KB per tile (4 and 16 measured no better)
  constexpr int64_t kTile = static_cast<int64_t>(kThreads) * kU;
  if (a.nkinds < 1 || a.nkinds > kMaxCopyKinds) return set_error(USP_ERR_INVALID_ARG, "internal: %d copy kinds", a.nkinds);
  a.tile_prefix[0] = 0;
  for (int k = 0; k < a.nkinds; ++k) {
    a.seg_tiles[k] = (a.rows[k] * a.nv + kTile - 1) / kTile;
    a.tile_prefix[k + 1] = a.tile_prefix[k] + a.outer * a.seg_tiles[k];
  }
  const int64_t tiles = a.tile_prefix[a.nkinds];
  if (tiles == 0) return USP_OK;
  copy_rows_kernel<kU><<<grid_for(tiles), kThreads, 0, s>>>(a);
  count_launch();
  return cuda_check(cudaGetLastError(), "segmented row copy launch");
}

int launch_reduce_scatter_rows(const RowsArgs& a, int vec_bytes, int dtype, cudaStream_t s) {
  switch (dtype) {
    case USP_BF16: return reduce_e<__nv_bfloat16>(a, vec_bytes, s);
    case USP_FP16: return reduce_e<__half>(a, vec_bytes, s);
    case USP_FP32: return reduce_e<float>(a, vec_bytes, s);
    default: return set_error(USP_ERR_DTYPE, "unknown dtype %d", dtype);
  }
}

int read_rows_bounds(uint32_t* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_rows_bounds, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_check(e, "read rows bounds word");
  if (reset) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_rows_bounds, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_check(e, "reset rows bounds word");
  }
  return USP_OK;
}

}  // namespace usp
