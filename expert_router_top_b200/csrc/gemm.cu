// gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// The expert computation of the Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE",
// section 核心原理), with the SwiGLU FFN form:
//   gate/up:  Act[r] = bf16( silu(X[r] W_gate[e]^T) * (X[r] W_up[e]^T) )   (K = H)
//   down:     Y[r]   = bf16( Act[r] W_down[e]^T )                           (K = I)
// for every row r of expert e, rows of one expert being contiguous (offsets[e] ..
// offsets[e+1]).  Only these two GEMMs are dense contractions on the path.
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: per 64-wide K block, one 128x64 A box and the B boxes
//               (gate/up: 128 gate rows + 128 up rows; down: 256 rows), 128-byte swizzle,
//               into a 4-stage shared-memory ring guarded by mbarriers.
//   warp 1      MMA issuer: allocates 512 TMEM columns (two 128x256 fp32 accumulators),
//               issues tcgen05.mma M=128 N=256 K=16 from one thread, commits each stage
//               back to the producer and each finished tile to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator rows (warp w reads TMEM lanes
//               32*(w%4)..+31), SwiGLU or plain conversion to bf16, predicated 16-byte
//               stores of the rows that belong to the tile's expert.  Double-buffered
//               TMEM lets the epilogue of tile i overlap the MMAs of tile i+1.
// Tiles are enumerated expert by expert, N tile by N tile, M tile fastest, so the CTAs
// running at the same time share their weight (B) tiles in L2.  A tile's rows past its
// expert's end are computed from whatever rows follow (or TMA zero fill) and never
// stored.  Every row's result depends only on that row, the weights and a fixed MMA
// sequence, so it does not depend on where the row sits in a tile or a chunk: outputs are
// bit-identical for any chunking.
#include <stdio.h>

#include "device.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK, STAGES = kGemmStages;
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KB
constexpr uint32_t kBBytes = BN * BK * 2;  // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators
constexpr uint32_t kIdesc = umma_idesc_bf16_f32(BM, BN);
constexpr int kMaxE = 1024;

struct KParams {
  const int32_t* offsets;
  __nv_bfloat16* out;
  uint32_t* status;
  int32_t E;
  int32_t n_tiles;   // N tiles per expert
  int32_t num_kb;    // K blocks
  int32_t out_cols;  // valid output columns
  int32_t b_rows;    // B rows per expert
  int32_t up_off;    // row offset of W_up inside one expert's W_gate_up (= I)
  int32_t total_tiles;
};

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kCtlBytes = 256;
static_assert(sizeof(SmemCtl) <= kCtlBytes, "control block");
constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + STAGES * kStageBytes + kCtlBytes +
                              2 * (kMaxE + 1) * sizeof(int32_t);

struct Tile {
  int32_t e, n, m;
};

__device__ __forceinline__ Tile decode_tile(int32_t L, const int32_t* tile_start,
                                            const int32_t* off, int32_t E, int32_t n_tiles) {
  // largest e with tile_start[e] <= L; that expert has at least one tile
  int32_t lo = 0, hi = E - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= L) lo = mid;
    else hi = mid - 1;
  }
  const int32_t mt = (off[lo + 1] - off[lo] + BM - 1) / BM;
  const int32_t local = L - tile_start[lo];
  Tile t;
  t.e = lo;
  t.n = local / mt;
  t.m = local - t.n * mt;
  (void)n_tiles;
  return t;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const KParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + STAGES * kStageBytes);
  int32_t* off = reinterpret_cast<int32_t*>(smem + STAGES * kStageBytes + kCtlBytes);
  int32_t* tile_start = off + (kMaxE + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t E = p.E;

  // ---- set-up: expert offsets, tile prefix, barriers, TMEM ----
  for (int32_t i = threadIdx.x; i <= E; i += kGemmThreads) off[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], 4 * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 2) {
    // exclusive prefix of tiles per expert: lane l covers experts [l*per, (l+1)*per)
    const int32_t per = (E + 31) / 32;
    const int32_t e0 = lane * per, e1 = min(E, e0 + per);
    int32_t sum = 0;
    for (int32_t e = e0; e < e1; ++e) sum += ((off[e + 1] - off[e] + BM - 1) / BM) * p.n_tiles;
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int32_t run = incl - sum;
    for (int32_t e = e0; e < e1; ++e) {
      tile_start[e] = run;
      run += ((off[e + 1] - off[e] + BM - 1) / BM) * p.n_tiles;
    }
    if (lane == 31) tile_start[E] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int* abort = &ctl->abort;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_last();    // weights: reused by many M tiles
      const uint64_t pol_a = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bits, for the abort drain
      bool ok = true;
      for (int32_t L = blockIdx.x; L < p.total_tiles && ok; L += gridDim.x) {
        const Tile t = decode_tile(L, tile_start, off, E, p.n_tiles);
        const int32_t row0 = off[t.e] + t.m * BM;
        const int32_t brow = t.e * p.b_rows + t.n * (kSwiGLU ? BN / 2 : BN);
        for (int32_t kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
          uint8_t* a_dst = sA + stage * kABytes;
          uint8_t* b_dst = sB + stage * kBBytes;
          tma_load_2d(a_dst, &tmA, &ctl->full[stage], kb * BK, row0, pol_a);
          if (kSwiGLU) {
            tma_load_2d(b_dst, &tmB, &ctl->full[stage], kb * BK, brow, pol_w);
            tma_load_2d(b_dst + kBBytes / 2, &tmB, &ctl->full[stage], kb * BK, brow + p.up_off,
                        pol_w);
          } else {
            tma_load_2d(b_dst, &tmB, &ctl->full[stage], kb * BK, brow, pol_w);
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wait (bounded) for the copies already issued, so none lands after exit
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_drain(&ctl->full[s], (armed_parity >> s) & 1u, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      int32_t it = 0;
      for (int32_t L = blockIdx.x; L < p.total_tiles && ok; L += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t tphase = (it >> 1) & 1;
        if (!mbar_wait(&ctl->tempty[buf], tphase ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int32_t kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // advance 16 bf16 = 32 bytes along K inside the 128-byte swizzled row
            umma_bf16(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                      sw128_kmajor_desc(b_addr + kk * 32), kIdesc, (kb | kk) != 0);
          }
          issued = true;
          umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[buf]);
      }
      if (!ok && issued) {
        // every MMA issued so far must finish before TMEM is released
        umma_commit(&ctl->drain);
        mbar_drain(&ctl->drain, 0, 100000000ull);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    int32_t it = 0;
    for (int32_t L = blockIdx.x; L < p.total_tiles; L += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t tphase = (it >> 1) & 1;
      if (!mbar_wait(&ctl->tfull[buf], tphase, abort, p.status)) break;
      tc_fence_after();
      const Tile t = decode_tile(L, tile_start, off, E, p.n_tiles);
      const int32_t rows_valid = off[t.e + 1] - off[t.e] - t.m * BM;
      const bool row_ok = r < rows_valid;
      const int64_t row = (int64_t)off[t.e] + t.m * BM + r;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * BN;
      if (kSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < (BN / 2) / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld_32cols(t_row + c * 32, g);
          tmem_ld_32cols(t_row + BN / 2 + c * 32, u);
          tmem_ld_wait2(g, u);
          const int32_t col0 = t.n * (BN / 2) + c * 32;
          if (row_ok) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              const float a0 = g0 / (1.0f + __expf(-g0)) * u0;
              const float a1 = g1 / (1.0f + __expf(-g1)) * u1;
              packed[i] = pack_bf16x2(a0, a1);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * p.out_cols + col0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (col0 + v * 8 < p.out_cols)
                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                    packed[4 * v + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t acc[32];
          tmem_ld_32cols(t_row + c * 32, acc);
          tmem_ld_wait(acc);
          const int32_t col0 = t.n * BN + c * 32;
          if (row_ok) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = pack_bf16x2(__uint_as_float(acc[2 * i]), __uint_as_float(acc[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * p.out_cols + col0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (col0 + v * 8 < p.out_cols)
                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                    packed[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix with a box of
// box_rows x 64 columns and the 128-byte swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int32_t cols, int32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int64_t gemm_total_tiles(const int32_t* counts_host, int32_t E, int32_t out_cols, bool swiglu) {
  const int32_t bn = swiglu ? BN / 2 : BN;
  const int64_t n_tiles = (out_cols + bn - 1) / bn;
  int64_t m_tiles = 0;
  for (int32_t e = 0; e < E; ++e) m_tiles += (counts_host[e] + BM - 1) / BM;
  return m_tiles * n_tiles;
}

cudaError_t launch_grouped_gemm(const GemmArgs& a, bool swiglu, int num_sms, cudaStream_t s,
                                int* err_detail) {
  *err_detail = 0;
  if (a.total_tiles <= 0) return cudaSuccess;
  if (a.total_tiles > 0x7fffffff || a.E > kMaxE) {
    *err_detail = 1;
    return cudaErrorInvalidValue;
  }
  CUtensorMap mA, mB;
  const int32_t bn = swiglu ? BN / 2 : BN;
  if (!make_map(&mA, a.A, a.rows, a.K, BM) ||
      !make_map(&mB, a.B, (int64_t)a.E * a.b_rows, a.K, swiglu ? BN / 2 : BN)) {
    *err_detail = 2;
    return cudaErrorInvalidValue;
  }
  KParams p;
  p.offsets = a.offsets;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.status = a.status;
  p.E = a.E;
  p.n_tiles = (a.out_cols + bn - 1) / bn;
  p.num_kb = (a.K + BK - 1) / BK;
  p.out_cols = a.out_cols;
  p.b_rows = a.b_rows;
  p.up_off = swiglu ? a.out_cols : 0;
  p.total_tiles = (int32_t)a.total_tiles;
  const int grid = (int)(a.total_tiles < num_sms ? a.total_tiles : num_sms);
  cudaError_t e;
  if (swiglu) {
    e = cudaFuncSetAttribute(grouped_gemm_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<true><<<grid, kGemmThreads, kSmemBytes, s>>>(mA, mB, p);
  } else {
    e = cudaFuncSetAttribute(grouped_gemm_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<false><<<grid, kGemmThreads, kSmemBytes, s>>>(mA, mB, p);
  }
  return cudaGetLastError();
}

}  // namespace moe
