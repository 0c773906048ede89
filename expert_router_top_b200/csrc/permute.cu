// permute.cu -- dispatch (permute) and weighted combine (unpermute) of one chunk.
//
// Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE"), section 核心原理: permute
// groups the token copies by expert before the expert computation, unpermute restores
// token order and merges the k copies afterwards; section 一张专业时序图 lists
// top_k_weights among the inputs split per chunk, and the merge is weighted by them.
//
// Both kernels are HBM-bound row movers: one warp per token, 16-byte (8 x bf16) vector
// accesses, every lane a different 16-byte column of the row, so each warp instruction
// touches 512 contiguous bytes.
//   permute:   reads token row t once, writes its k copies   ->  (1 + k) * H * 2 bytes
//   unpermute: reads the k expert rows of token t, writes one ->  (k + 1) * H * 2 bytes
#include "device.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRowThreads = 256;          // 8 tokens per CTA
constexpr int kTokPerCta = kRowThreads / 32;

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ uint32_t g_range_flags;  // checks build: a row index outside its buffer was seen

// The call's metadata found an expert index out of range: its rows are not to be used.
__device__ __forceinline__ bool guarded_out(const uint32_t* guard) {
  return guard && (*reinterpret_cast<const volatile uint32_t*>(guard) & MOE_DEV_BAD_INDEX);
}

// X[dst[t*k+j]] = hidden[t] for every j < k.  The warp loads the next U x 512 bytes of the
// token row before it stores the k copies of the current ones, so the row's (usually cold)
// reads stay in flight while the stores issue.
template <int U>
__global__ void __launch_bounds__(kRowThreads) permute_kernel(const uint4* __restrict__ hidden,
                                                              const int32_t* __restrict__ dst,
                                                              int64_t Tc, int32_t H8, int32_t k,
                                                              uint4* __restrict__ X,
                                                              int64_t rows_cap,
                                                              const uint32_t* guard) {
  const int64_t t = (int64_t)blockIdx.x * kTokPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= Tc || guarded_out(guard)) return;
  const int32_t d_lane = lane < k ? dst[t * k + lane] : 0;
  const uint4* src = hidden + t * H8;
  uint4 cur[U], nxt[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int32_t v = u * 32 + lane;
    cur[u] = v < H8 ? ldg_stream(src + v) : make_uint4(0, 0, 0, 0);
  }
  for (int32_t v0 = 0; v0 < H8; v0 += 32 * U) {
    const int32_t v1 = v0 + 32 * U;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int32_t v = v1 + u * 32 + lane;
      nxt[u] = v < H8 ? ldg_stream(src + v) : make_uint4(0, 0, 0, 0);
    }
    for (int j = 0; j < k; ++j) {
      const int32_t d = __shfl_sync(0xffffffffu, d_lane, j);
      if (!check_row(d, rows_cap, &g_range_flags)) continue;
      uint4* row = X + (int64_t)d * H8;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int32_t v = v0 + u * 32 + lane;
        if (v < H8) row[v] = cur[u];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) cur[u] = nxt[u];
  }
}

// out[t] = bf16( sum_{j<k} w[t*k+j] * Y[dst[t*k+j]] ), fp32 accumulation, j ascending.
template <int U>
__global__ void __launch_bounds__(kRowThreads) unpermute_kernel(const uint4* __restrict__ Y,
                                                                const int32_t* __restrict__ dst,
                                                                const float* __restrict__ w,
                                                                int64_t Tc, int32_t H8, int32_t k,
                                                                uint4* __restrict__ out,
                                                                int64_t rows_cap,
                                                                const uint32_t* guard) {
  const int64_t t = (int64_t)blockIdx.x * kTokPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= Tc || guarded_out(guard)) return;
  const int32_t d_lane = lane < k ? dst[t * k + lane] : 0;
  const float w_lane = lane < k ? w[t * k + lane] : 0.f;
  for (int32_t v0 = 0; v0 < H8; v0 += 32 * U) {
    float acc[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int32_t d = __shfl_sync(0xffffffffu, d_lane, j);
      const float wj = __shfl_sync(0xffffffffu, w_lane, j);
      if (!check_row(d, rows_cap, &g_range_flags)) continue;
      const uint4* row = Y + (int64_t)d * H8;
      uint4 y[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int32_t v = v0 + u * 32 + lane;
        y[u] = v < H8 ? ldg_stream(row + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t q[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[u][2 * i] = fmaf(wj, bf16lo(q[i]), acc[u][2 * i]);
          acc[u][2 * i + 1] = fmaf(wj, bf16hi(q[i]), acc[u][2 * i + 1]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int32_t v = v0 + u * 32 + lane;
      if (v < H8) {
        uint4 o;
        o.x = pack_bf16x2(acc[u][0], acc[u][1]);
        o.y = pack_bf16x2(acc[u][2], acc[u][3]);
        o.z = pack_bf16x2(acc[u][4], acc[u][5]);
        o.w = pack_bf16x2(acc[u][6], acc[u][7]);
        out[t * H8 + v] = o;
      }
    }
  }
}

// The same combine with k fixed at compile time: a warp issues the loads of all k rows'
// 16-byte vectors -- for k < 8 of 8 / k vectors per lane -- before the first FMA, so about
// 8 x 512 bytes per warp are in flight instead of one row's, and loops over tokens
// (grid-stride) so that the grid can be sized to the GPU.  The arithmetic is the kernel's
// above: acc = 0, then acc = fma(w_j, y_j, acc) for j = 0 .. k-1, so both give the same bits.
// At most 64 registers per thread (four CTAs per SM): the combine that runs beside a grouped
// GEMM must fit on the SM sub-partitions next to the GEMM's warps.
template <int KT>
__global__ void __launch_bounds__(kRowThreads, 4) unpermute_k_kernel(const uint4* __restrict__ Y,
                                                                     const int32_t* __restrict__ dst,
                                                                     const float* __restrict__ w,
                                                                     int64_t Tc, int32_t H8,
                                                                     uint4* __restrict__ out,
                                                                     int64_t rows_cap,
                                                                     const uint32_t* guard) {
  constexpr int V = KT >= 8 ? 1 : 8 / KT;  // vectors per lane per pass
  const int lane = threadIdx.x & 31;
  if (guarded_out(guard)) return;
  const int64_t n_warps = (int64_t)gridDim.x * kTokPerCta;
  for (int64_t t = (int64_t)blockIdx.x * kTokPerCta + (threadIdx.x >> 5); t < Tc; t += n_warps) {
    const int32_t d_lane = lane < KT ? dst[t * KT + lane] : 0;
    const float w_lane = lane < KT ? w[t * KT + lane] : 0.f;
    int32_t row[KT];  // row index (a 32-bit register each; the address is formed per load)
    float wj[KT];
    bool ok[KT];
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      const int32_t d = __shfl_sync(0xffffffffu, d_lane, j);
      wj[j] = __shfl_sync(0xffffffffu, w_lane, j);
      ok[j] = check_row(d, rows_cap, &g_range_flags);
      row[j] = ok[j] ? d : 0;
    }
    for (int32_t v0 = lane; v0 < H8; v0 += 32 * V) {
      uint4 y[V][KT];
#pragma unroll
      for (int u = 0; u < V; ++u)
#pragma unroll
        for (int j = 0; j < KT; ++j) {
          const int32_t v = v0 + 32 * u;
          y[u][j] = v < H8 ? ldg_stream(Y + (int64_t)row[j] * H8 + v) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int u = 0; u < V; ++u) {
        const int32_t v = v0 + 32 * u;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < KT; ++j) {
          if (!ok[j]) continue;
          const uint32_t q[4] = {y[u][j].x, y[u][j].y, y[u][j].z, y[u][j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(wj[j], bf16lo(q[i]), acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj[j], bf16hi(q[i]), acc[2 * i + 1]);
          }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        if (v < H8) out[t * H8 + v] = o;
      }
    }
  }
}

inline unsigned grid_for(int64_t Tc) { return (unsigned)((Tc + kTokPerCta - 1) / kTokPerCta); }

#ifndef MOE_UNPERM_CTAS_PER_SM
#define MOE_UNPERM_CTAS_PER_SM 4  // grid of the compile-time-k combine: CTAs per SM
#endif

int num_sms_cached() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& v = n[dev & 63];
  if (v <= 0 && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    v = 148;
  return v;
}

template <int KT>
cudaError_t launch_unpermute_k(const void* Y, const int32_t* dst, const float* w, int64_t Tc,
                               int32_t H, void* out, int64_t rows_cap, cudaStream_t s,
                               int ctas_per_sm, const uint32_t* guard) {
  const int64_t cap =
      (int64_t)num_sms_cached() * (ctas_per_sm > 0 ? ctas_per_sm : MOE_UNPERM_CTAS_PER_SM);
  const int64_t need = grid_for(Tc);
  unpermute_k_kernel<KT><<<(unsigned)(need < cap ? need : cap), kRowThreads, 0, s>>>(
      static_cast<const uint4*>(Y), dst, w, Tc, H / 8, static_cast<uint4*>(out), rows_cap,
      guard);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_permute(const void* hidden, const int32_t* dst, int64_t Tc, int32_t H,
                           int32_t k, void* X, int64_t rows_cap, cudaStream_t s,
                           const uint32_t* guard) {
  if (Tc <= 0) return cudaSuccess;
  permute_kernel<4><<<grid_for(Tc), kRowThreads, 0, s>>>(
      static_cast<const uint4*>(hidden), dst, Tc, H / 8, k, static_cast<uint4*>(X), rows_cap,
      guard);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* Y, const int32_t* dst, const float* w, int64_t Tc,
                             int32_t H, int32_t k, void* out, int64_t rows_cap, cudaStream_t s,
                             int ctas_per_sm, const uint32_t* guard) {
  if (Tc <= 0) return cudaSuccess;
#if MOE_UNPERM_CTAS_PER_SM > 0
  switch (k) {
    case 1: return launch_unpermute_k<1>(Y, dst, w, Tc, H, out, rows_cap, s, ctas_per_sm, guard);
    case 2: return launch_unpermute_k<2>(Y, dst, w, Tc, H, out, rows_cap, s, ctas_per_sm, guard);
    case 4: return launch_unpermute_k<4>(Y, dst, w, Tc, H, out, rows_cap, s, ctas_per_sm, guard);
    case 6: return launch_unpermute_k<6>(Y, dst, w, Tc, H, out, rows_cap, s, ctas_per_sm, guard);
    case 8: return launch_unpermute_k<8>(Y, dst, w, Tc, H, out, rows_cap, s, ctas_per_sm, guard);
    default: break;
  }
#endif
  unpermute_kernel<2><<<grid_for(Tc), kRowThreads, 0, s>>>(
      static_cast<const uint4*>(Y), dst, w, Tc, H / 8, k, static_cast<uint4*>(out), rows_cap,
      guard);
  return cudaGetLastError();
}

uint32_t checks_take_permute() {
  uint32_t v = 0, zero = 0;
  if (!MOE_CHECKS) return 0;
  cudaMemcpyFromSymbol(&v, g_range_flags, sizeof v);
  cudaMemcpyToSymbol(g_range_flags, &zero, sizeof zero);
  return v;
}

}  // namespace moe
