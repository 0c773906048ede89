// noalloc.cu -- moe_metadata_noalloc: the batched metadata pass without any allocation.
//
// Some callers cannot allocate device memory at the point where they need the routing
// metadata: a runtime whose device memory is owned entirely by its own caching
// allocator and that forbids out-of-band cudaMalloc/cudaFree (cudaFree also synchronizes
// the whole device), a latency-critical serving path that cannot pay for an allocation,
// or a plugin that is handed only its inputs and outputs.  For them this entry point
// keeps its scratch (status word, per-chunk counts, offsets and splits, per-tile
// histograms) in one fixed file-scope device array instead of a caller workspace, and
// copies the results to the host through a fixed host array; it calls no allocating
// routine (no cudaMalloc/cudaFree, no cudaMallocHost, no stream or event creation).
//
// The array is shared by every call on a device and keeps the previous call's contents;
// each call clears the status word it relies on and overwrites everything else it reads.
// Calls whose work overlaps on the GPU (two streams, two host threads) race on it.
#include <string.h>

#include <mutex>

#include "device.cuh"
#include "internal.h"
#include "moe.h"

namespace {

constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
constexpr int kStatusWords = 4;
constexpr int kMaxDevices = 64;

// The scratch array: one per device that loads this library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// The packed {status, counts, splits} block comes back to the host here.
static int32_t g_host_pack[kScratchBytes / sizeof(int32_t)];

void* g_scratch_dev[kMaxDevices];  // device address of g_noalloc_scratch, per device
std::mutex g_noalloc_mu;

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Plan {
  int32_t n, G, tile_tokens, tiles_per_chunk;
  int64_t t_chunk;
  size_t packed_bytes, offsets, hist, total;
};

Plan plan(int64_t T, int32_t k, int32_t E, int32_t ep_groups, int32_t num_chunks) {
  Plan p;
  p.n = num_chunks > 0 ? num_chunks : 1;
  p.G = ep_groups > 0 ? ep_groups : 1;
  p.t_chunk = (T + p.n - 1) / p.n;
  p.tile_tokens = moe::meta_tile_tokens(k);
  p.tiles_per_chunk = (int32_t)((p.t_chunk + p.tile_tokens - 1) / p.tile_tokens);
  if (p.tiles_per_chunk < 1) p.tiles_per_chunk = 1;
  p.packed_bytes = sizeof(int32_t) * (kStatusWords + (size_t)p.n * E + (size_t)p.n * p.G);
  p.offsets = al256(p.packed_bytes);
  p.hist = p.offsets + al256(sizeof(int32_t) * (size_t)p.n * (E + 1));
  p.total = p.hist + al256(sizeof(int32_t) * (size_t)p.n * p.tiles_per_chunk * E);
  return p;
}

// Per-device set-up: the device address of the scratch array, looked up once with the
// device current.  In host code the array's name is only a host-side stand-in; a kernel
// must be given this address.
moe_status_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_scratch_dev[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return MOE_ERR_CUDA;
    g_scratch_dev[dev] = ptr;
  }
  *out = g_scratch_dev[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status_t moe_metadata_noalloc(const int32_t* top_k_index, int64_t T, int32_t k, int32_t E,
                                  int32_t ep_groups, int32_t num_chunks, int32_t* send_splits,
                                  int32_t* recv_splits, int32_t* expert_counts,
                                  int64_t* chunk_bounds, int32_t* dst_rows, int32_t* src_tokens,
                                  void* stream) {
  if (T < 0 || k <= 0 || E <= 0 || ep_groups < 0 || num_chunks < 0) return MOE_ERR_ARG;
  const int32_t G = ep_groups > 0 ? ep_groups : 1;
  if (k > E || E % G != 0) return MOE_ERR_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK || num_chunks > MOE_MAX_CHUNKS)
    return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (!send_splits || !recv_splits || !expert_counts || !chunk_bounds) return MOE_ERR_ARG;
  if (T > 0 && (!top_k_index || !dst_rows)) return MOE_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(top_k_index) % 4 || reinterpret_cast<uintptr_t>(dst_rows) % 4 ||
      reinterpret_cast<uintptr_t>(src_tokens) % 4)
    return MOE_ERR_ALIGN;
  const Plan p = plan(T, k, E, ep_groups, num_chunks);
  if (p.total > kScratchBytes) return MOE_ERR_WORKSPACE;  // beyond the fixed scratch array
  moe_chunk_bounds(T, num_chunks, chunk_bounds);
  if (T == 0) {
    memset(send_splits, 0, sizeof(int32_t) * (size_t)p.n * G);
    memset(recv_splits, 0, sizeof(int32_t) * (size_t)p.n * G);
    memset(expert_counts, 0, sizeof(int32_t) * (size_t)p.n * E);
    return MOE_OK;
  }
  void* base = nullptr;
  moe_status_t st = scratch_address(&base);
  if (st != MOE_OK) return st;
  unsigned char* ws = static_cast<unsigned char*>(base);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  moe::MetaArgs a;
  a.idx = top_k_index;
  a.T = T;
  a.k = k;
  a.E = E;
  a.G = G;
  a.n_chunks = p.n;
  a.t_chunk = p.t_chunk;
  a.tile_tokens = p.tile_tokens;
  a.tiles_per_chunk = p.tiles_per_chunk;
  a.hist = reinterpret_cast<int32_t*>(ws + p.hist);
  a.dst = dst_rows;
  a.src_tok = src_tokens;
  int32_t* packed = reinterpret_cast<int32_t*>(ws);
  a.status = reinterpret_cast<uint32_t*>(packed);
  a.counts = packed + kStatusWords;
  a.splits = a.counts + (size_t)p.n * E;
  a.offsets = reinterpret_cast<int32_t*>(ws + p.offsets);
  // the status words must start at zero (the previous call may have left a flag in them):
  // the metadata kernel clears them
  a.status_words = kStatusWords;
  if (moe::launch_metadata(a, s) != cudaSuccess) return MOE_ERR_CUDA;
  // the single device-to-host copy, into the fixed host array
  if (cudaMemcpyAsync(g_host_pack, packed, p.packed_bytes, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  const uint32_t status = static_cast<uint32_t>(g_host_pack[0]);
  if (status & moe::MOE_DEV_BAD_INDEX) return MOE_ERR_INDEX;
  const int32_t* counts = g_host_pack + kStatusWords;
  const int32_t* splits = counts + (size_t)p.n * E;
  memcpy(expert_counts, counts, sizeof(int32_t) * (size_t)p.n * E);
  memcpy(send_splits, splits, sizeof(int32_t) * (size_t)p.n * G);
  memcpy(recv_splits, splits, sizeof(int32_t) * (size_t)p.n * G);
  return MOE_OK;
}

}  // extern "C"
