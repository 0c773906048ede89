// metadata.cu -- batched pre-dispatch metadata for every chunk in one pass.
//
// Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE"), section 一张专业时序图: the
// send/receive splits, per-rank token counts and local per-expert token counts of all
// chunks are produced together, so that one host copy serves every chunk.  Section
// 核心原理: permute groups each token copy by its destination expert; here the order is
// experts ascending (so virtual EP groups ascending: "rank-major") and, inside one expert,
// the flat copy index t*k+j ascending, which makes the permutation deterministic and
// independent of the number of chunks.
//
// Three small kernels, no atomics on the data path (only on the error flag):
//   rank:     per tile of copies, a stable in-tile rank of every copy within its expert
//             (warp match + per-warp histograms) and the tile's expert histogram;
//   count:    per (chunk, expert), an exclusive scan of the tile histograms over the
//             chunk's tiles -> each tile's base inside the expert, and the chunk counts;
//   finalize: per tile, the chunk's expert offsets (scan of counts), the final row
//             dst = offset[e] + tile base[e] + in-tile rank, the inverse map src_tok, and
//             (first tile of each chunk) the offsets and group splits.
#include "device.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = kMetaThreads / 32;

struct TileSpan {
  int64_t chunk_tok0;  // first token of the chunk
  int64_t tok0;        // first token of the tile
  int32_t slots;       // copies in the tile (0 for a tile past the chunk's end)
};

__device__ __forceinline__ TileSpan tile_span(const MetaArgs& a, int32_t tile) {
  const int32_t c = tile / a.tiles_per_chunk;
  const int32_t lt = tile - c * a.tiles_per_chunk;
  TileSpan s;
  s.chunk_tok0 = (int64_t)c * a.t_chunk;
  int64_t chunk_end = s.chunk_tok0 + a.t_chunk;
  if (chunk_end > a.T) chunk_end = a.T;
  s.tok0 = s.chunk_tok0 + (int64_t)lt * a.tile_tokens;
  int64_t tok1 = s.tok0 + a.tile_tokens;
  if (tok1 > chunk_end) tok1 = chunk_end;
  s.slots = tok1 > s.tok0 ? (int32_t)((tok1 - s.tok0) * a.k) : 0;
  return s;
}

// Slots [w*seg, (w+1)*seg) of the tile belong to warp w; seg is a multiple of 32.
__device__ __forceinline__ int32_t warp_segment(int32_t slots) {
  return ((slots + kWarps * 32 - 1) / (kWarps * 32)) * 32;
}

__global__ void __launch_bounds__(kMetaThreads) meta_rank_kernel(MetaArgs a) {
  extern __shared__ int32_t sm[];
  int32_t* whist = sm;                       // [kWarps][E]
  int32_t* lrank = sm + kWarps * a.E;        // [kMetaSlotsPerTile]
  const int32_t tile = blockIdx.x;
  const TileSpan ts = tile_span(a, tile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * a.E; i += kMetaThreads) whist[i] = 0;
  __syncthreads();

  const int32_t seg = warp_segment(ts.slots);
  const int32_t* idx = a.idx + ts.tok0 * a.k;
  int32_t* my_hist = whist + warp * a.E;
  const int32_t s_begin = warp * seg;
  const int32_t s_end = min(ts.slots, s_begin + seg);
  for (int32_t base = s_begin; base < s_end; base += 32) {
    const int32_t s = base + lane;
    int32_t e = -1;
    if (s < s_end) {
      e = idx[s];
      if (e < 0 || e >= a.E) {
        atomicOr(a.status, MOE_DEV_BAD_INDEX);
        e = -1;
      }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    int32_t prior = 0;
    if (e >= 0) {
      prior = my_hist[e];
      lrank[s] = prior + __popc(peers & lanemask_lt());
    }
    __syncwarp();
    if (e >= 0 && (__ffs(peers) - 1) == lane) my_hist[e] = prior + __popc(peers);
    __syncwarp();
  }
  __syncthreads();

  // exclusive prefix over warps, per expert; the total is the tile histogram
  for (int32_t e = threadIdx.x; e < a.E; e += kMetaThreads) {
    int32_t run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int32_t v = whist[w * a.E + e];
      whist[w * a.E + e] = run;
      run += v;
    }
    a.hist[(int64_t)tile * a.E + e] = run;
  }
  __syncthreads();

  int32_t* dst = a.dst + ts.tok0 * a.k;
  for (int32_t s = threadIdx.x; s < ts.slots; s += kMetaThreads) {
    const int32_t e = idx[s];
    if (e < 0 || e >= a.E) continue;
    dst[s] = whist[(s / seg) * a.E + e] + lrank[s];  // rank inside the tile
  }
}

__global__ void __launch_bounds__(kMetaThreads) meta_count_kernel(MetaArgs a) {
  const int32_t c = blockIdx.x;
  const int32_t e = blockIdx.y * kMetaThreads + threadIdx.x;
  if (e >= a.E) return;
  int32_t* h = a.hist + (int64_t)c * a.tiles_per_chunk * a.E + e;
  int32_t run = 0;
  // 8 tiles at a time: the 8 loads are issued together instead of one round trip per tile
  for (int32_t lt0 = 0; lt0 < a.tiles_per_chunk; lt0 += 8) {
    int32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = lt0 + u < a.tiles_per_chunk ? h[(int64_t)(lt0 + u) * a.E] : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (lt0 + u < a.tiles_per_chunk) h[(int64_t)(lt0 + u) * a.E] = run;
      run += v[u];
    }
  }
  a.counts[(int64_t)c * a.E + e] = run;
}

// Block-wide exclusive scan of counts[0..E) into off[0..E] (off[E] = total).
__device__ void block_exclusive_scan(const int32_t* counts, int32_t E, int32_t* off,
                                     int32_t* warp_tot) {
  const int per = (E + kMetaThreads - 1) / kMetaThreads;  // <= 4 for E <= 1024
  const int e0 = threadIdx.x * per;
  int32_t local = 0;
  for (int i = 0; i < per; ++i)
    if (e0 + i < E) local += counts[e0 + i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int32_t v = warp_tot[w];
      warp_tot[w] = run;
      run += v;
    }
    off[E] = run;
  }
  __syncthreads();
  int32_t run = warp_tot[warp] + incl - local;
  for (int i = 0; i < per; ++i) {
    if (e0 + i < E) {
      off[e0 + i] = run;
      run += counts[e0 + i];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kMetaThreads) meta_finalize_kernel(MetaArgs a) {
  extern __shared__ int32_t sm[];
  int32_t* off = sm;                  // [E+1]
  int32_t* warp_tot = sm + a.E + 1;   // [kWarps]
  const int32_t tile = blockIdx.x;
  const int32_t c = tile / a.tiles_per_chunk;
  const int32_t lt = tile - c * a.tiles_per_chunk;
  const TileSpan ts = tile_span(a, tile);
  block_exclusive_scan(a.counts + (int64_t)c * a.E, a.E, off, warp_tot);

  if (lt == 0) {
    int32_t* offsets = a.offsets + (int64_t)c * (a.E + 1);
    for (int32_t e = threadIdx.x; e <= a.E; e += kMetaThreads) offsets[e] = off[e];
    const int32_t per_group = a.E / a.G;
    for (int32_t g = threadIdx.x; g < a.G; g += kMetaThreads)
      a.splits[(int64_t)c * a.G + g] = off[(g + 1) * per_group] - off[g * per_group];
  }

  const int32_t* idx = a.idx + ts.tok0 * a.k;
  const int32_t* base = a.hist + (int64_t)tile * a.E;
  int32_t* dst = a.dst + ts.tok0 * a.k;
  int32_t* src = a.src_tok ? a.src_tok + ts.chunk_tok0 * a.k : nullptr;
  const int32_t tok_in_chunk0 = (int32_t)(ts.tok0 - ts.chunk_tok0);
  // 8 slots per thread at a time: their index and rank loads are issued together
  for (int32_t s0 = threadIdx.x; s0 < ts.slots; s0 += 8 * kMetaThreads) {
    int32_t e[8], rk[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int32_t sl = s0 + u * kMetaThreads;
      e[u] = sl < ts.slots ? idx[sl] : -1;
      rk[u] = sl < ts.slots ? dst[sl] : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int32_t sl = s0 + u * kMetaThreads;
      if (e[u] < 0 || e[u] >= a.E) continue;
      const int32_t r = off[e[u]] + base[e[u]] + rk[u];
      dst[sl] = r;
      if (src)
        src[r] = (int32_t)((a.src_relative ? 0 : ts.chunk_tok0) + tok_in_chunk0 + sl / a.k);
    }
  }
}

}  // namespace

cudaError_t launch_metadata(const MetaArgs& a, cudaStream_t s) {
  const int32_t n_tiles = a.n_chunks * a.tiles_per_chunk;
  const size_t rank_smem = sizeof(int32_t) * ((size_t)kWarps * a.E + kMetaSlotsPerTile);
  const size_t fin_smem = sizeof(int32_t) * ((size_t)a.E + 1 + kWarps);
  // rank_smem <= (8 * 1024 + 2048) * 4 B = 40 KB: within the default 48 KB limit
  meta_rank_kernel<<<n_tiles, kMetaThreads, rank_smem, s>>>(a);
  meta_count_kernel<<<dim3(a.n_chunks, (a.E + kMetaThreads - 1) / kMetaThreads), kMetaThreads, 0,
                      s>>>(a);
  meta_finalize_kernel<<<n_tiles, kMetaThreads, fin_smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
