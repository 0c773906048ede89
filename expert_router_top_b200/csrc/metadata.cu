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
// One cooperative kernel in three phases separated by grid-wide barriers (its CTAs loop over
// the tiles, so that every CTA of the grid is resident), no atomics on the data path (only
// on the error flag):
//   rank:     per tile of copies, a stable in-tile rank of every copy within its expert
//             (warp match + per-warp histograms) and the tile's expert histogram;
//   count:    per (chunk, expert), an exclusive scan of the tile histograms over the
//             chunk's tiles -> each tile's base inside the expert, and the chunk counts;
//   finalize: per tile, the chunk's expert offsets (scan of counts), the final row
//             dst = offset[e] + tile base[e] + in-tile rank, the inverse map src_tok, and
//             (first tile of each chunk) the offsets and group splits.
// The status words are cleared by the kernel itself, before the first barrier; a bad index
// seen in the rank phase is recorded after the last one.
#include <cooperative_groups.h>

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

// Returns whether the tile holds an expert index outside [0, E).
__device__ bool meta_rank_tile(const MetaArgs& a, int32_t tile, int32_t* sm) {
  int32_t* whist = sm;                       // [kWarps][E]
  int32_t* lrank = sm + kWarps * a.E;        // [kMetaSlotsPerTile]: e << 16 | rank, or -1
  const TileSpan ts = tile_span(a, tile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool bad = false;
  for (int i = threadIdx.x; i < kWarps * a.E; i += kMetaThreads) whist[i] = 0;
  __syncthreads();

  const int32_t seg = warp_segment(ts.slots);
  const int32_t* idx = a.idx + ts.tok0 * a.k;
  int32_t* my_hist = whist + warp * a.E;
  const int32_t s_begin = warp * seg;
  const int32_t s_end = min(ts.slots, s_begin + seg);
  // the warp's expert indices, all loads issued before the first use (seg <= 32 * kIt)
  constexpr int kIt = kMetaSlotsPerTile / kMetaThreads;
  static_assert(kMetaSlotsPerTile % kMetaThreads == 0, "whole segments");
  int32_t ev[kIt];
#pragma unroll
  for (int u = 0; u < kIt; ++u) {
    const int32_t s = s_begin + u * 32 + lane;
    ev[u] = s < s_end ? idx[s] : -1;
  }
#pragma unroll
  for (int u = 0; u < kIt; ++u) {
    const int32_t s = s_begin + u * 32 + lane;
    if (s_begin + u * 32 >= s_end) break;  // warp-uniform
    int32_t e = ev[u];
    if (s < s_end && (e < 0 || e >= a.E)) {
      bad = true;
      lrank[s] = -1;
      e = -1;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    int32_t prior = 0;
    if (e >= 0) {
      prior = my_hist[e];
      lrank[s] = e << 16 | (prior + __popc(peers & lanemask_lt()));
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
    const int32_t v = lrank[s];
    if (v < 0) continue;
    dst[s] = whist[(s / seg) * a.E + (v >> 16)] + (v & 0xffff);  // rank inside the tile
  }
  __syncthreads();  // the shared arrays are reused by the next tile
  return bad;
}

// Column (c, e) of the tile histograms, one warp: exclusive scan over the chunk's tiles, in
// place, 32 tiles per round (a lane per tile, warp scan), and the chunk's count of expert e.
__device__ void meta_count_column(const MetaArgs& a, int32_t c, int32_t e, int lane) {
  int32_t* h = a.hist + (int64_t)c * a.tiles_per_chunk * a.E + e;
  int32_t run = 0;
  for (int32_t lt0 = 0; lt0 < a.tiles_per_chunk; lt0 += 32) {
    const int32_t lt = lt0 + lane;
    const int32_t v = lt < a.tiles_per_chunk ? h[(int64_t)lt * a.E] : 0;
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lt < a.tiles_per_chunk) h[(int64_t)lt * a.E] = run + incl - v;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) a.counts[(int64_t)c * a.E + e] = run;
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

__device__ void meta_finalize_tile(const MetaArgs& a, int32_t tile, int32_t* sm) {
  int32_t* off = sm;                  // [E+1]
  int32_t* warp_tot = sm + a.E + 1;   // [kWarps]
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
  __syncthreads();  // off is reused by the next tile
}

__global__ void __launch_bounds__(kMetaThreads) meta_kernel(MetaArgs a) {
  extern __shared__ int32_t sm[];
  cooperative_groups::grid_group grid = cooperative_groups::this_grid();
  const int32_t n_tiles = a.n_chunks * a.tiles_per_chunk;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.status_words; i += kMetaThreads) a.status[i] = 0;
  bool bad = false;
  for (int32_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x)
    bad |= meta_rank_tile(a, tile, sm);
  grid.sync();
  const int32_t cols = a.n_chunks * a.E;
  const int warp = threadIdx.x >> 5;
  for (int32_t i = blockIdx.x * kWarps + warp; i < cols; i += gridDim.x * kWarps)
    meta_count_column(a, i / a.E, i % a.E, threadIdx.x & 31);
  grid.sync();
  for (int32_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x)
    meta_finalize_tile(a, tile, sm);
  if (bad) atomicOr(a.status, MOE_DEV_BAD_INDEX);  // after the clear: two barriers later
}

}  // namespace

cudaError_t launch_metadata(const MetaArgs& a, cudaStream_t s) {
  const int32_t n_tiles = a.n_chunks * a.tiles_per_chunk;
  const size_t rank_smem = sizeof(int32_t) * ((size_t)kWarps * a.E + kMetaSlotsPerTile);
  const size_t fin_smem = sizeof(int32_t) * ((size_t)a.E + 1 + kWarps);
  // <= (8 * 1024 + 2048) * 4 B = 40 KB: within the default 48 KB limit
  const size_t smem = rank_smem > fin_smem ? rank_smem : fin_smem;
  // every CTA of a cooperative grid must be resident: at most the device's capacity at the
  // largest shared-memory size (E = 1024, the most experts), looked up once per device; the
  // CTAs loop over the tiles
  constexpr int kMaxDevices = 64;
  static int cap_of[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (cap_of[dev] <= 0) {
    constexpr size_t kMaxSmem = sizeof(int32_t) * ((size_t)kWarps * 1024 + kMetaSlotsPerTile);
    static_assert(kMaxSmem <= 48 * 1024, "within the default dynamic shared-memory limit");
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, meta_kernel, kMetaThreads,
                                                        kMaxSmem);
    if (e != cudaSuccess) return e;
    cap_of[dev] = sms * per_sm;
  }
  const int64_t cap = cap_of[dev];
  if (cap <= 0 || smem > sizeof(int32_t) * ((size_t)kWarps * 1024 + kMetaSlotsPerTile))
    return cudaErrorInvalidConfiguration;
  const int grid = (int)(n_tiles < cap ? (n_tiles > 0 ? n_tiles : 1) : cap);
  MetaArgs args = a;
  void* params[] = {&args};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(meta_kernel), dim3(grid),
                                     dim3(kMetaThreads), params, smem, s);
}

}  // namespace moe
