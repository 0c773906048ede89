// ep.cu -- expert parallelism over several GPUs with the exchange fused into the row kernels.
//
// Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE"), sections 一张专业时序图 (per
// chunk: dispatch All-to-All -> experts -> combine All-to-All, the two chunks of a pair
// overlapping) and 操作指南 (expert_parallel_size): the experts are split over W ranks,
// rank d owning experts [d E/W, (d+1) E/W), and each chunk's token copies travel to the
// rank of their expert and back.
//
// On B200s joined by NVLink/NVSwitch every GPU can store to and load from its peers'
// memory directly, so the exchange needs no separate collective or staging copy: the
// dispatch kernel writes each token copy's row straight into its row of the owning rank's
// receive buffer (peer stores), and the combine kernel reads the expert outputs from there
// (peer loads) while it forms the weighted sum.  Plain 16-byte loads and stores only: no
// TMA, no multicast.
//
// Receive layout on rank d (the input of its grouped GEMMs): local expert by local expert,
// and inside one expert the source ranks in ascending order, each source's rows in that
// source's own stable (t, j) order.  Every rank knows where its rows go from the per-chunk
// expert counts of all ranks (one all-gather of W x E integers per chunk, the pages'
// AllGather of the routing counts): moe_ep_plan turns them into one row offset per
// (destination, expert, source), and the device kernels add it to the chunk-local row that
// moe_metadata gives each copy.
#include <string.h>

#include "device.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

constexpr int kEpThreads = 256;  // 8 tokens per CTA, one warp per token
constexpr int kEpTokPerCta = kEpThreads / 32;

__device__ uint32_t g_ep_range_flags;  // checks build: a receive row outside its buffer

__device__ __forceinline__ uint4 ld_nc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// recv[owner(e)][dst[t k + j] + delta[e]] = hidden[t] for every copy (t, j), e = idx[t k + j].
__global__ void __launch_bounds__(kEpThreads) ep_dispatch_kernel(
    const uint4* __restrict__ hidden, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ dst, const int32_t* __restrict__ delta, uint4* const* recv,
    int64_t Tc, int32_t H8, int32_t k, int32_t E, int32_t e_per_rank, int64_t rows_cap) {
  const int64_t t = (int64_t)blockIdx.x * kEpTokPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= Tc) return;
  int32_t row_lane = -1, rank_lane = 0;
  if (lane < k) {
    const int32_t e = idx[t * k + lane];
    if (e >= 0 && e < E) {  // an index the metadata flagged is skipped, never followed
      row_lane = dst[t * k + lane] + delta[e];
      rank_lane = e / e_per_rank;
    }
  }
  const uint4* src = hidden + t * H8;
  for (int32_t v0 = 0; v0 < H8; v0 += 64) {
    uint4 val[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int32_t v = v0 + u * 32 + lane;
      if (v < H8) val[u] = ld_nc(src + v);
    }
    for (int j = 0; j < k; ++j) {
      const int32_t row = __shfl_sync(0xffffffffu, row_lane, j);
      const int32_t rk = __shfl_sync(0xffffffffu, rank_lane, j);
      // always bounded (a receive buffer may be another GPU's memory); the checks build
      // also records the violation
      if (row < 0 || row >= rows_cap) {
        check_row(row, rows_cap, &g_ep_range_flags);
        continue;
      }
      uint4* out = recv[rk] + (int64_t)row * H8;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int32_t v = v0 + u * 32 + lane;
        if (v < H8) out[v] = val[u];
      }
    }
  }
}

// out[t] = bf16( sum_{j<k} w[t k + j] * Y[owner(e)][dst[t k + j] + delta[e]] ), fp32, j
// ascending: the arithmetic of the single-GPU unpermute, reading the rows from their rank.
__global__ void __launch_bounds__(kEpThreads) ep_combine_kernel(
    const uint4* const* expert_rows, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ dst, const int32_t* __restrict__ delta,
    const float* __restrict__ w, int64_t Tc, int32_t H8, int32_t k, int32_t E,
    int32_t e_per_rank, int64_t rows_cap, uint4* __restrict__ out) {
  const int64_t t = (int64_t)blockIdx.x * kEpTokPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= Tc) return;
  int32_t row_lane = -1, rank_lane = 0;
  float w_lane = 0.f;
  if (lane < k) {
    const int32_t e = idx[t * k + lane];
    if (e >= 0 && e < E) {
      row_lane = dst[t * k + lane] + delta[e];
      rank_lane = e / e_per_rank;
    }
    w_lane = w[t * k + lane];
  }
  for (int32_t v0 = 0; v0 < H8; v0 += 32) {
    const int32_t v = v0 + lane;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t row = __shfl_sync(0xffffffffu, row_lane, j);
      const int32_t rk = __shfl_sync(0xffffffffu, rank_lane, j);
      const float wj = __shfl_sync(0xffffffffu, w_lane, j);
      if (row < 0 || row >= rows_cap) {
        check_row(row, rows_cap, &g_ep_range_flags);
        continue;
      }
      if (v >= H8) continue;
      const uint4 y = ld_nc(expert_rows[rk] + (int64_t)row * H8 + v);
      const uint32_t q[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(wj, bf16lo(q[i]), acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj, bf16hi(q[i]), acc[2 * i + 1]);
      }
    }
    if (v < H8) {
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      out[t * H8 + v] = o;
    }
  }
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the runtime's driver entry point (no link against libcuda).
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(ptr);
  }
  return fn;
}

moe_status_t check_ep(int64_t Tc, int32_t H, int32_t k, int32_t E, int32_t W, int64_t rows_cap) {
  if (Tc < 0 || H <= 0 || H % 8 != 0 || k <= 0 || E <= 0 || W <= 0 || rows_cap < 0)
    return MOE_ERR_ARG;
  if (k > E || E % W != 0) return MOE_ERR_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK || W > MOE_EP_MAX_RANKS) return MOE_ERR_UNSUPPORTED;
  if (Tc * (int64_t)k >= (int64_t)1 << 31 || rows_cap >= (int64_t)1 << 31)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace

uint32_t checks_take_ep() {
  uint32_t v = 0, zero = 0;
  if (!MOE_CHECKS) return 0;
  cudaMemcpyFromSymbol(&v, g_ep_range_flags, sizeof v);
  cudaMemcpyToSymbol(g_ep_range_flags, &zero, sizeof zero);
  return v;
}

}  // namespace moe

extern "C" {

moe_status_t moe_ep_plan(const int32_t* counts_all, int32_t W, int32_t rank, int32_t E,
                         int32_t* send_delta, int32_t* recv_offsets) {
  if (!counts_all || !send_delta || !recv_offsets) return MOE_ERR_ARG;
  if (W <= 0 || E <= 0 || E % W != 0 || rank < 0 || rank >= W) return MOE_ERR_ARG;
  if (E > MOE_MAX_EXPERTS || W > MOE_EP_MAX_RANKS) return MOE_ERR_UNSUPPORTED;
  const int32_t El = E / W;
  for (int64_t i = 0; i < (int64_t)W * E; ++i)
    if (counts_all[i] < 0) return MOE_ERR_ARG;
  // as a source: copy (t, j) of expert e sits at chunk-local row offsets_rank[e] + r (the
  // metadata's expert-major layout) and goes to row base(owner(e), e, rank) + r
  int64_t own_off = 0;  // offsets_rank[e], the running sum of this rank's counts
  for (int32_t e = 0; e < E; ++e) {
    const int32_t d = e / El;
    int64_t base = 0;  // rows of d's receive buffer before (e, source 0)
    for (int32_t e2 = d * El; e2 < e; ++e2)
      for (int32_t s = 0; s < W; ++s) base += counts_all[(int64_t)s * E + e2];
    for (int32_t s = 0; s < rank; ++s) base += counts_all[(int64_t)s * E + e];
    const int64_t delta = base - own_off;
    if (delta < INT32_MIN || delta > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    send_delta[e] = (int32_t)delta;
    own_off += counts_all[(int64_t)rank * E + e];
  }
  // as a destination: where each local expert's rows start, and the total
  int64_t run = 0;
  for (int32_t el = 0; el <= El; ++el) {
    if (run > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    recv_offsets[el] = (int32_t)run;
    if (el == El) break;
    for (int32_t s = 0; s < W; ++s) run += counts_all[(int64_t)s * E + (int64_t)rank * El + el];
  }
  return MOE_OK;
}

moe_status_t moe_ep_dispatch(const void* hidden, const int32_t* top_k_index,
                             const int32_t* dst_rows, const int32_t* send_delta,
                             void* const* recv_rows, int64_t Tc, int32_t H, int32_t k, int32_t E,
                             int32_t W, int64_t rows_cap, void* stream) {
  moe_status_t st = moe::check_ep(Tc, H, k, E, W, rows_cap);
  if (st != MOE_OK) return st;
  if (Tc == 0) return MOE_OK;
  if (!hidden || !top_k_index || !dst_rows || !send_delta || !recv_rows) return MOE_ERR_ARG;
  if (!moe::al16(hidden)) return MOE_ERR_ALIGN;
  const unsigned grid = (unsigned)((Tc + moe::kEpTokPerCta - 1) / moe::kEpTokPerCta);
  moe::ep_dispatch_kernel<<<grid, moe::kEpThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(hidden), top_k_index, dst_rows, send_delta,
      reinterpret_cast<uint4* const*>(recv_rows), Tc, H / 8, k, E, E / W, rows_cap);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ep_combine(void* const* expert_rows, const int32_t* top_k_index,
                            const int32_t* dst_rows, const int32_t* send_delta,
                            const float* top_k_weights, int64_t Tc, int32_t H, int32_t k,
                            int32_t E, int32_t W, int64_t rows_cap, void* out, void* stream) {
  moe_status_t st = moe::check_ep(Tc, H, k, E, W, rows_cap);
  if (st != MOE_OK) return st;
  if (Tc == 0) return MOE_OK;
  if (!expert_rows || !top_k_index || !dst_rows || !send_delta || !top_k_weights || !out)
    return MOE_ERR_ARG;
  if (!moe::al16(out)) return MOE_ERR_ALIGN;
  const unsigned grid = (unsigned)((Tc + moe::kEpTokPerCta - 1) / moe::kEpTokPerCta);
  moe::ep_combine_kernel<<<grid, moe::kEpThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4* const*>(expert_rows), top_k_index, dst_rows, send_delta,
      top_k_weights, Tc, H / 8, k, E, E / W, rows_cap, static_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ipc_handle(const void* dev_ptr, void* handle, int64_t* offset) {
  if (!dev_ptr || !handle || !offset) return MOE_ERR_ARG;
  CUdeviceptr base = 0;
  size_t size = 0;
  moe::AddressRangeFn range = moe::address_range_fn();
  if (!range || range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return MOE_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return MOE_ERR_CUDA;
  static_assert(sizeof(h) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
  memcpy(handle, &h, sizeof h);
  *offset = (int64_t)(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return MOE_OK;
}

moe_status_t moe_ipc_open(const void* handle, int64_t offset, void** dev_ptr) {
  if (!handle || !dev_ptr || offset < 0) return MOE_ERR_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
    return MOE_ERR_CUDA;
  *dev_ptr = static_cast<uint8_t*>(base) + offset;
  return MOE_OK;
}

moe_status_t moe_ipc_close(void* dev_ptr, int64_t offset) {
  if (!dev_ptr || offset < 0) return MOE_ERR_ARG;
  return cudaIpcCloseMemHandle(static_cast<uint8_t*>(dev_ptr) - offset) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // extern "C"
