// backward.cu -- backward pass of the chunked MoE layer, with the expert computation
// recomputed per pair of chunks (the pipeline's unit).
//
// The Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE") trains through this layer:
// the backward pass mirrors the forward chunk pipeline (section 一张专业时序图, the last
// paragraph on the timing diagram) and the expert computation may be recomputed to keep the
// activation peak low (chunk_moe_recompute, sections 一组关键公式 and 操作指南).  For one
// copy (t, j) routed to expert e, with x = hidden[t]:
//   g = W_gate x, u = W_up x, h = silu(g) u                      (recomputed)
//   a = W_down^T dout[t];  d_w[t][j] = <dout[t], W_down h> = <a, h>;  dh = w[t][j] a
//   du = dh silu(g);  dg = dh u silu'(g);  dX = W_gate^T dg + W_up^T du
//   d_hidden[t] = sum_j dX;  dW_down[e] += dout[t] (w[t][j] h)^T;  dW_gate|up[e] += dg|du x^T
// The output y = W_down h of the copy is never formed: its only use in the backward pass,
// d_w, is the same inner product taken on the I side, where the SwiGLU-backward epilogue
// already holds both a and h.
//
// Backward buffers hold each expert's rows of one unit padded to a multiple of 64 (zero
// rows), so that the weight-gradient GEMMs reduce over an expert's rows in whole 64-row K
// blocks.  The helpers below speak of "chunks": the metadata's chunks, which the pipeline
// makes the pairs of the layer's chunks.
//
// The GEMMs run on one tcgen05 kernel (one CTA per SM, TMA producer warp, one MMA thread,
// four epilogue warps, 4-stage ring, double-buffered TMEM, as the forward kernel) in four
// modes:
//   kRawGU    [g u] = X W_gate_up^T           A rows K-major, B K-major   epilogue: g, u, w h
//   kDSwiGLU  a = dY W_down (dY = dout rows)  B MN-major                  epilogue: dg, du,
//                                                                         partial <a, h>
//   kDPlain   dX = [dg du] W_gate_up          B MN-major                  epilogue: bf16 store
//   kWGrad    dW[e] += S_A[e]^T S_B[e]        A and B MN-major, K = rows  epilogue: TMA fp32
//             (K = the expert's padded rows of one pair of chunks)      store / add-reduce
// MN-major operands use the 128-byte-swizzled MN-major canonical layout: 64-element MN
// blocks of 64 K rows x 128 B (8 KB apart: the leading byte offset), 8-row K groups 1 KB
// apart (the stride byte offset); one MMA K step of 16 advances 2 KB.
#include <string.h>

#include <vector>

#include "device.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
// Epilogue warps per mode: eight (two per TMEM lane quarter, each taking half of the tile's
// columns) where the epilogue does per-element math; four for the weight gradients, whose
// epilogue is a TMA store per block and whose staging buffer is sized for four warps.
template <int kMode>
struct Cfg {
  static constexpr int kEpi = kMode == 3 ? 4 : 8;
  static constexpr int kThreads = 64 + 32 * kEpi;
};
constexpr uint32_t kABytes = BM * BK * 2, kBBytes = BN * BK * 2, kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 2 * BN;
constexpr int kMaxE = 1024;
constexpr int kPadRows = 64;  // backward rows of one expert are padded to this multiple

enum Mode { kRawGU = 0, kDSwiGLU = 1, kDPlain = 2, kWGrad = 3 };

__device__ uint32_t g_range_flags;  // checks build: a row index outside its buffer was seen

struct BParams {
  const int32_t* offsets;  // padded expert row offsets [E+1] (multiples of 64)
  uint32_t* status;
  int32_t E;
  int32_t m_tiles;   // kWGrad: M tiles per expert
  int32_t n_tiles;   // N tiles per expert
  int32_t num_kb;    // row-grouped modes: K blocks
  int32_t M;         // kWGrad: rows of the gradient
  int32_t N;         // output columns
  int32_t I;         // gate/up split of 2I-wide tensors
  int32_t b_rows;    // rows of one expert's weight matrix in B
  int32_t total_tiles;
  __nv_bfloat16* out0;      // kRawGU: GU [rows][2I]; kDSwiGLU: [dg du] [rows][2I]
                            // (may be aux: each block is read before it is stored); kDPlain: [rows][N]
  __nv_bfloat16* out1;      // kRawGU: Act = w h [rows][I]
  const __nv_bfloat16* aux; // kDSwiGLU: GU [rows][2I]
  const float* wrow;        // kRawGU, kDSwiGLU: routing weight of each row [rows] (0 on pads)
  float* dwp;               // kDSwiGLU: [rows][dw_slots] partial <a, h> of each (tile column,
                            // epilogue warp column half), or nullptr
  int32_t dw_slots;         // kDSwiGLU: 2 * n_tiles
  float* acc;               // kWGrad: [E][M][N] fp32 (written through tmC)
  const int32_t* first;     // kWGrad: [E] first unit (pair of chunks) with rows of each expert
  int32_t chunk;            // kWGrad: the unit of this launch (store where first == chunk)
  int64_t rows;             // checks build: rows of the A / output buffers
};

struct Ctl {
  uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kCtlBytes = 256;
static_assert(sizeof(Ctl) <= kCtlBytes, "control block");
// kWGrad output staging: one 32 x 32 fp32 box (4 KB, 128-byte swizzled) per epilogue warp
constexpr uint32_t kOutBoxBytes = 32 * 32 * 4;
constexpr uint32_t kOutBytes = 4 * kOutBoxBytes;
constexpr size_t kSmem =
    1024 + STAGES * kStageBytes + kOutBytes + kCtlBytes + 2 * (kMaxE + 1) * 4;
static_assert(kSmem <= 232448, "shared memory per CTA");

__host__ __device__ constexpr uint32_t idesc(bool a_mn, bool b_mn) {
  return umma_idesc_bf16_f32(BM, BN) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
}

// MN-major operand descriptor (128-byte swizzle): LBO = 8 KB between 64-element MN blocks,
// SBO = 1 KB between 8-row K groups, version 1, swizzle mode 2.
__device__ __forceinline__ uint64_t mn_desc(uint32_t addr) {
  return static_cast<uint64_t>((addr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(8192 >> 4) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// A tile: expert e, column tile n, row tile m.
struct Tile {
  int32_t e, m, n;
};

template <int kMode>
__device__ __forceinline__ Tile decode(int32_t L, const int32_t* ts, const int32_t* off,
                                       int32_t E, const BParams& p) {
  int32_t lo = 0, hi = E - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (ts[mid] <= L) lo = mid;
    else hi = mid - 1;
  }
  const int32_t local = L - ts[lo];
  Tile t;
  t.e = lo;
  if (kMode == kWGrad) {
    t.m = local / p.n_tiles;
    t.n = local - t.m * p.n_tiles;
  } else {
    const int32_t mt = (off[lo + 1] - off[lo] + BM - 1) / BM;
    t.n = local / mt;
    t.m = local - t.n * mt;
  }
  return t;
}

// One epilogue warp's 32 rows x 32 bf16 columns (lane i holds row i as 16 packed pairs)
// through 2 KB of shared memory: 16-byte chunk c of row r sits at c ^ ((r >> 1) & 3), which
// keeps both the row-wise writes and the 8-rows-per-instruction reads free of bank
// conflicts.  Row rr of the block goes to out + (row0 + rr) * ld + col0; rows at or past
// nrows and columns at or past ncols are not written.
__device__ __forceinline__ void store_block_staged(const uint32_t (&pk)[16], uint8_t* wbuf,
                                                   int lane, __nv_bfloat16* out, int64_t row0,
                                                   int32_t ld, int32_t col0, int32_t ncols,
                                                   int32_t nrows, int64_t rows_cap) {
  uint8_t* mine = wbuf + lane * 64;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(mine + ((c ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  __syncwarp();
  const int seg = lane & 3;
  const int32_t col = col0 + seg * 8;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int rr = pass * 8 + (lane >> 2);
    const uint4 v = *reinterpret_cast<const uint4*>(wbuf + rr * 64 + ((seg ^ ((rr >> 1) & 3)) << 4));
    if (rr < nrows && col < ncols && check_row(row0 + rr, rows_cap, &g_range_flags))
      *reinterpret_cast<uint4*>(out + (row0 + rr) * ld + col) = v;
  }
  __syncwarp();
}

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int kMode>
__global__ void __launch_bounds__(Cfg<kMode>::kThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const BParams p) {
  constexpr bool kAmn = kMode == kWGrad;
  constexpr bool kBmn = kMode != kRawGU;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  uint8_t* sOut = smem + STAGES * kStageBytes;  // 1024-byte aligned
  Ctl* ctl = reinterpret_cast<Ctl*>(sOut + kOutBytes);
  int32_t* off = reinterpret_cast<int32_t*>(sOut + kOutBytes + kCtlBytes);
  int32_t* ts = off + (kMaxE + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t E = p.E;

  constexpr int kEpi = Cfg<kMode>::kEpi;
  for (int32_t i = threadIdx.x; i <= E; i += Cfg<kMode>::kThreads) off[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], kEpi * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 2) {  // exclusive prefix of tiles per expert
    const int32_t per = (E + 31) / 32;
    const int32_t e0 = lane * per, e1 = min(E, e0 + per);
    auto tiles_of = [&](int32_t e) -> int32_t {
      const int32_t rows = off[e + 1] - off[e];
      if (kMode == kWGrad) return rows > 0 ? p.m_tiles * p.n_tiles : 0;
      return (rows + BM - 1) / BM * p.n_tiles;
    };
    int32_t sum = 0;
    for (int32_t e = e0; e < e1; ++e) sum += tiles_of(e);
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int32_t run = incl - sum;
    for (int32_t e = e0; e < e1; ++e) {
      ts[e] = run;
      run += tiles_of(e);
    }
    if (lane == 31) ts[E] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int* abort = &ctl->abort;

  if (warp == 0) {
    if (lane == 0) {  // ---------------- TMA producer ----------------
      const uint64_t pol = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int32_t L = blockIdx.x; L < p.total_tiles && ok; L += gridDim.x) {
        const Tile t = decode<kMode>(L, ts, off, E, p);
        const int32_t nkb = kMode == kWGrad ? (off[t.e + 1] - off[t.e]) / BK : p.num_kb;
        for (int32_t kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
          uint8_t* a = sA + stage * kABytes;
          uint8_t* b = sB + stage * kBBytes;
          uint64_t* bar = &ctl->full[stage];
          if (kMode == kWGrad) {
            const int32_t r0 = off[t.e] + kb * BK;
            for (int q = 0; q < 2; ++q) tma_load_2d(a + q * 8192, &tmA, bar, t.m * BM + q * 64, r0, pol);
            for (int q = 0; q < 4; ++q) tma_load_2d(b + q * 8192, &tmB, bar, t.n * BN + q * 64, r0, pol);
          } else {
            const int32_t row0 = off[t.e] + t.m * BM;
            tma_load_2d(a, &tmA, bar, kb * BK, row0, pol);
            if (kMode == kRawGU) {
              const int32_t brow = t.e * p.b_rows + t.n * (BN / 2);
              tma_load_2d(b, &tmB, bar, kb * BK, brow, pol);
              tma_load_2d(b + kBBytes / 2, &tmB, bar, kb * BK, brow + p.I, pol);
            } else {  // MN-major weights: K rows of expert e, 4 blocks of 64 output columns
              const int32_t krow = t.e * p.b_rows + kb * BK;
              for (int q = 0; q < 4; ++q)
                tma_load_2d(b + q * 8192, &tmB, bar, t.n * BN + q * 64, krow, pol);
            }
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok)
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_drain(&ctl->full[s], (armed_parity >> s) & 1u, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      int32_t it = 0;
      for (int32_t L = blockIdx.x; L < p.total_tiles && ok; L += gridDim.x, ++it) {
        const Tile t = decode<kMode>(L, ts, off, E, p);
        const int32_t nkb = kMode == kWGrad ? (off[t.e + 1] - off[t.e]) / BK : p.num_kb;
        const int buf = it & 1;
        if (!mbar_wait(&ctl->tempty[buf], ((it >> 1) & 1) ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int32_t kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = kAmn ? mn_desc(a_addr + kk * 2048) : kmajor_desc<128>(a_addr + kk * 32);
            const uint64_t bd = kBmn ? mn_desc(b_addr + kk * 2048) : kmajor_desc<128>(b_addr + kk * 32);
            umma_bf16(d_tmem, ad, bd, idesc(kAmn, kBmn), (kb | kk) != 0);
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
        umma_commit(&ctl->drain);
        mbar_drain(&ctl->drain, 0, 100000000ull);
      }
    }
  } else {  // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    // column half of this warp when two warps share a lane quarter
    const int part = (warp - 2) >> 2;
    constexpr int kParts = kEpi / 4;
    constexpr int kC = BN / 32 / kParts;        // 32-column blocks per warp
    constexpr int kCgu = BN / 2 / 32 / kParts;  // gate/up column-block pairs per warp
    const int r = q * 32 + lane;  // accumulator row (TMEM lane)
    int32_t it = 0;
    for (int32_t L = blockIdx.x; L < p.total_tiles; L += gridDim.x, ++it) {
      const int buf = it & 1;
      const Tile t = decode<kMode>(L, ts, off, E, p);
      // kDSwiGLU: the saved g and u of this thread's row, one 32-column block ahead of the
      // accumulator; the first block is requested before the accumulator is ready
      uint4 gq[4], uq[4];
      const int32_t rows_here = off[t.e + 1] - off[t.e] - t.m * BM;
      const int64_t row_g = (int64_t)off[t.e] + t.m * BM + r;
      const __nv_bfloat16* aux = p.aux;
      auto load_aux = [&](int c, uint4 (&g)[4], uint4 (&u)[4]) {
        const uint4* gu4 = reinterpret_cast<const uint4*>(aux + row_g * 2 * p.I);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const int32_t cc = t.n * BN + c * 32 + v4 * 8;
          if (r < rows_here && cc < p.I) {
            g[v4] = __ldg(gu4 + cc / 8);
            u[v4] = __ldg(gu4 + (p.I + cc) / 8);
          } else {
            g[v4] = make_uint4(0, 0, 0, 0);
            u[v4] = g[v4];
          }
        }
      };
      if (kMode == kDSwiGLU) load_aux(part * kC, gq, uq);
      // routing weight of this thread's row (0 for rows past the expert's)
      float wr = 0.f;
      if ((kMode == kRawGU || kMode == kDSwiGLU) && r < rows_here &&
          check_row(row_g, p.rows, &g_range_flags))
        wr = __ldg(p.wrow + row_g);
      if (!mbar_wait(&ctl->tfull[buf], (it >> 1) & 1, abort, p.status)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * BN;
      if (kMode == kWGrad) {
        // Each warp owns accumulator rows q*32..q*32+31: per 32-column block it stages the
        // 32 x 32 fp32 block in shared memory (16-byte chunk i of row `lane` at i ^ (lane % 8),
        // the 128-byte swizzle of the tensor map) and one lane stores it -- the expert's first
        // pair of chunks with rows -- or adds it into dW with one TMA reduction.  Each element
        // of dW gets one store or add per pair, in pair order.
        uint8_t* box = sOut + q * kOutBoxBytes;
        const int32_t m0 = t.m * BM + q * 32;
        const bool store = p.first[t.e] == p.chunk;
#pragma unroll 1
        for (int c = part * kC; c < (part + 1) * kC; ++c) {
          uint32_t v[32];
          tmem_ld_32cols(t_row + c * 32, v);
          if (lane == 0) bulk_wait_read_all();  // the previous box has left shared memory
          __syncwarp();
          tmem_ld_wait(v);
          float4* row4 = reinterpret_cast<float4*>(box + lane * 128);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            row4[i ^ (lane & 7)] =
                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          fence_async_smem();
          __syncwarp();
          const int32_t col0 = t.n * BN + c * 32;
          if (lane == 0 && m0 < p.M && col0 < p.N) {
            if (store) tma_store_3d(&tmC, box, col0, m0, t.e);
            else tma_reduce_add_3d(&tmC, box, col0, m0, t.e);
            bulk_commit();
          }
        }
      } else {
        // rows of this warp's 32-row block that belong to the expert (the others are the
        // next expert's) and the block's first output row
        const int32_t rows_valid = off[t.e + 1] - off[t.e] - t.m * BM;
        const int32_t nrows = rows_valid - q * 32;
        const int64_t row0w = (int64_t)off[t.e] + t.m * BM + q * 32;
        const int64_t cap = p.rows;
        __nv_bfloat16* o0 = p.out0;
        __nv_bfloat16* o1 = p.out1;
        uint8_t* wbuf = sOut + (warp - 2) * 2048;  // 2 KB per epilogue warp
        if (kMode == kRawGU) {
#pragma unroll 1
          for (int c = part * kCgu; c < (part + 1) * kCgu; ++c) {
            uint32_t g[32], u[32];
            tmem_ld_32cols(t_row + c * 32, g);
            tmem_ld_32cols(t_row + BN / 2 + c * 32, u);
            tmem_ld_wait2(g, u);
            const int32_t col0 = t.n * (BN / 2) + c * 32;
            if (nrows <= 0 || col0 >= p.I) continue;  // warp-uniform
            uint32_t pg[16], pu[16], ph[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              pg[i] = pack_bf16x2(g0, g1);
              pu[i] = pack_bf16x2(u0, u1);
              ph[i] = pack_bf16x2(wr * (silu_f(g0) * u0), wr * (silu_f(g1) * u1));
            }
            store_block_staged(pg, wbuf, lane, o0, row0w, 2 * p.I, col0, p.I, nrows, cap);
            store_block_staged(pu, wbuf, lane, o0 + p.I, row0w, 2 * p.I, col0, p.I, nrows, cap);
            store_block_staged(ph, wbuf, lane, o1, row0w, p.I, col0, p.I, nrows, cap);
          }
        } else {
          float dwa = 0.f;  // kDSwiGLU: <a, h> over this warp's columns, in column order
#pragma unroll 1
          for (int c = part * kC; c < (part + 1) * kC; ++c) {
            uint32_t v[32];
            tmem_ld_32cols(t_row + c * 32, v);
            uint4 gn[4], un[4];
            if (kMode == kDSwiGLU && c + 1 < (part + 1) * kC) load_aux(c + 1, gn, un);
            tmem_ld_wait(v);
            const int32_t col0 = t.n * BN + c * 32;
            const int32_t ncols = kMode == kDSwiGLU ? p.I : p.N;
            if (nrows <= 0 || col0 >= ncols) continue;  // warp-uniform
            if (kMode == kDSwiGLU) {
              uint32_t dg[16], du[16];
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                const uint32_t ga[4] = {gq[v4].x, gq[v4].y, gq[v4].z, gq[v4].w};
                const uint32_t ua[4] = {uq[v4].x, uq[v4].y, uq[v4].z, uq[v4].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float dgv[2], duv[2];
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const float gv = h ? bf16hi(ga[i]) : bf16lo(ga[i]);
                    const float uv = h ? bf16hi(ua[i]) : bf16lo(ua[i]);
                    const float a = __uint_as_float(v[v4 * 8 + 2 * i + h]);
                    const float sig = __fdividef(1.0f, 1.0f + __expf(-gv));
                    dwa = fmaf(gv * sig * uv, a, dwa);
                    const float dh = wr * a;
                    duv[h] = dh * gv * sig;
                    dgv[h] = dh * uv * (sig + gv * sig * (1.0f - sig));
                  }
                  dg[v4 * 4 + i] = pack_bf16x2(dgv[0], dgv[1]);
                  du[v4 * 4 + i] = pack_bf16x2(duv[0], duv[1]);
                }
              }
              store_block_staged(dg, wbuf, lane, o0, row0w, 2 * p.I, col0, p.I, nrows, cap);
              store_block_staged(du, wbuf, lane, o0 + p.I, row0w, 2 * p.I, col0, p.I, nrows,
                                 cap);
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                gq[v4] = gn[v4];
                uq[v4] = un[v4];
              }
            } else {  // kDPlain
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              store_block_staged(pk, wbuf, lane, o0, row0w, p.N, col0, p.N, nrows, cap);
            }
          }
          // every slot of a row of the expert is written, 0 where its columns are past I
          if (kMode == kDSwiGLU && p.dwp && r < rows_here &&
              check_row(row_g, cap, &g_range_flags))
            p.dwp[row_g * p.dw_slots + t.n * kParts + part] = dwa;
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->tempty[buf]);
    }
    if (kMode == kWGrad && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- row kernels ----------------------------------------------------------------------

constexpr int kRowThreads = 256;
constexpr int kTokPerCta = kRowThreads / 32;

// Padded expert offsets of every chunk: offp[c][e] = sum_{e' < e} roundup(counts[c][e'], 64).
__global__ void pad_offsets_kernel(const int32_t* counts, int32_t E, int32_t* offp) {
  if (threadIdx.x != 0) return;
  const int32_t c = blockIdx.x;
  int32_t run = 0;
  for (int32_t e = 0; e < E; ++e) {
    offp[(int64_t)c * (E + 1) + e] = run;
    run += (counts[(int64_t)c * E + e] + kPadRows - 1) / kPadRows * kPadRows;
  }
  offp[(int64_t)c * (E + 1) + E] = run;
}

// first[e] = the first chunk in which expert e has rows (n_chunks if none).
__global__ void first_chunk_kernel(const int32_t* counts, int32_t E, int32_t n_chunks,
                                   int32_t* first) {
  const int32_t e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  int32_t c = 0;
  while (c < n_chunks && counts[(int64_t)c * E + e] == 0) ++c;
  first[e] = c;
}

// Padded row of each copy of one chunk, dstp = dst - off[e] + offp[e], and the copy's
// routing weight at that row: wrow[dstp] = w.
__global__ void pad_rows_kernel(const int32_t* idx, const int32_t* dst, const int32_t* off,
                                const int32_t* offp, const float* w, int64_t n, int32_t* dstp,
                                float* wrow, int64_t rows_cap) {
  const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= n) return;
  const int32_t e = idx[s];
  const int32_t d = dst[s] - off[e] + offp[e];
  const bool in = check_row(d, rows_cap, &g_range_flags);
  dstp[s] = in ? d : 0;
  if (in) wrow[d] = w[s];
}

// Zero the pad rows of a padded row buffer: rows offp[e] + (off[e+1] - off[e]) .. offp[e+1]
// of each expert e (fewer than kPadRows per expert), the only rows the permutes leave
// unwritten that the GEMMs read; and, where wrow is given, the routing weight of those rows.
// One CTA per expert.
__global__ void __launch_bounds__(256)
    zero_pad_rows_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ offp,
                         int32_t E, int32_t H8, uint4* __restrict__ buf, float* __restrict__ wrow,
                         int64_t rows_cap) {
  for (int32_t e = blockIdx.x; e < E; e += gridDim.x) {
    const int64_t r0 = (int64_t)offp[e] + (off[e + 1] - off[e]);
    const int64_t r1 = offp[e + 1];
    if (wrow && r0 + threadIdx.x < r1 && check_row(r0 + threadIdx.x, rows_cap, &g_range_flags))
      wrow[r0 + threadIdx.x] = 0.f;  // fewer than kPadRows <= blockDim.x pad rows
    const int64_t n = (r1 - r0) * H8;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
      const int64_t r = r0 + i / H8;
      if (check_row(r, rows_cap, &g_range_flags)) buf[r * H8 + i % H8] = make_uint4(0, 0, 0, 0);
    }
  }
}

// d_w[t][j] = the sum, in slot order, of the dSwiGLU epilogue's partial inner products of
// the copy's row.  One thread per copy.
__global__ void dw_sum_kernel(const float* __restrict__ dwp, const int32_t* __restrict__ dstp,
                              int64_t n, int32_t slots, float* __restrict__ dw, int64_t rows_cap) {
  const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= n) return;
  const int32_t d = dstp[s];
  if (!check_row(d, rows_cap, &g_range_flags)) return;
  float acc = 0.f;
  for (int32_t i = 0; i < slots; ++i) acc += dwp[(int64_t)d * slots + i];
  dw[s] = acc;
}

// d_hidden[t] = bf16( sum_{j<k} dX[dstp(t,j)] ), fp32 in ascending j.
__global__ void __launch_bounds__(kRowThreads)
    sum_rows_kernel(const uint4* __restrict__ dX, const int32_t* __restrict__ dstp, int64_t Tc,
                    int32_t H8, int32_t k, uint4* __restrict__ out, int64_t rows_cap) {
  const int64_t t = (int64_t)blockIdx.x * kTokPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= Tc) return;
  for (int32_t v = lane; v < H8; v += 32) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      const int32_t d = dstp[t * k + j];
      if (!check_row(d, rows_cap, &g_range_flags)) continue;
      const uint4 x = dX[(int64_t)d * H8 + v];
      const uint32_t xa[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += bf16lo(xa[i]);
        acc[2 * i + 1] += bf16hi(xa[i]);
      }
    }
    out[t * H8 + v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                 pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

template <int kMode>
cudaError_t launch_mode(const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mC,
                        const BParams& p, int num_sms, cudaStream_t s) {
  if (p.total_tiles <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<kMode>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int grid = p.total_tiles < num_sms ? p.total_tiles : num_sms;
  bwd_gemm_kernel<kMode><<<grid, Cfg<kMode>::kThreads, kSmem, s>>>(mA, mB, mC, p);
  return cudaGetLastError();
}

inline unsigned row_grid(int64_t Tc) { return (unsigned)((Tc + kTokPerCta - 1) / kTokPerCta); }

}  // namespace

int bwd_pad_rows() { return kPadRows; }

int32_t bwd_dw_slots(int32_t I) {
  static_assert(Cfg<kDSwiGLU>::kEpi / 4 == 2, "two epilogue warps per lane quarter");
  return 2 * ((I + BN - 1) / BN);
}

cudaError_t launch_bwd_gemm(const BwdGemmArgs& a, int num_sms, cudaStream_t s) {
  if (a.E > kMaxE) return cudaErrorInvalidValue;
  // host tile count from the padded per-expert rows
  int64_t tiles = 0;
  // N tiles: kRawGU pairs 128 gate with 128 up columns per tile; the others are 256 wide
  const int32_t n_tiles = a.mode == kRawGU ? (a.I + BN / 2 - 1) / (BN / 2) : (a.N + BN - 1) / BN;
  for (int32_t e = 0; e < a.E; ++e) {
    const int64_t r = a.rows_pad_host[e];
    if (a.mode == kWGrad) tiles += r > 0 ? (int64_t)((a.M + BM - 1) / BM) * n_tiles : 0;
    else tiles += (r + BM - 1) / BM * n_tiles;
  }
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 0x7fffffff) return cudaErrorInvalidValue;
  CUtensorMap mA, mB, mC;
  const bool a_mn = a.mode == kWGrad;
  const bool b_mn = a.mode != kRawGU;
  if (!make_tma_2d_bf16(&mA, a.A, a.A_rows, a.A_cols, a_mn ? BK : BM) ||
      !make_tma_2d_bf16(&mB, a.B, a.B_rows, a.B_cols, b_mn ? BK : BN / 2))
    return cudaErrorInvalidValue;
  if (a.mode == kWGrad) {
    if (!a.acc || !a.first || !make_tma_3d_f32(&mC, a.acc, a.E, a.M, a.N))
      return cudaErrorInvalidValue;
  } else {
    mC = mA;  // unused
  }
  BParams p;
  p.offsets = a.offsets;
  p.status = a.status;
  p.E = a.E;
  p.m_tiles = (a.M + BM - 1) / BM;
  p.n_tiles = n_tiles;
  p.num_kb = (a.K + BK - 1) / BK;
  p.M = a.M;
  p.N = a.N;
  p.I = a.I;
  p.b_rows = a.b_rows;
  p.total_tiles = (int32_t)tiles;
  p.out0 = static_cast<__nv_bfloat16*>(a.out0);
  p.out1 = static_cast<__nv_bfloat16*>(a.out1);
  p.aux = static_cast<const __nv_bfloat16*>(a.aux);
  p.wrow = a.wrow;
  p.dwp = a.dwp;
  p.dw_slots = a.mode == kDSwiGLU ? 2 * n_tiles : 0;
  if ((a.mode == kRawGU || a.mode == kDSwiGLU) && !a.wrow) return cudaErrorInvalidValue;
  p.acc = a.acc;
  p.first = a.first;
  p.chunk = a.chunk;
  p.rows = a.A_rows;
  switch (a.mode) {
    case kRawGU: return launch_mode<kRawGU>(mA, mB, mC, p, num_sms, s);
    case kDSwiGLU: return launch_mode<kDSwiGLU>(mA, mB, mC, p, num_sms, s);
    case kDPlain: return launch_mode<kDPlain>(mA, mB, mC, p, num_sms, s);
    case kWGrad: return launch_mode<kWGrad>(mA, mB, mC, p, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_pad_offsets(const int32_t* counts, int32_t E, int32_t n_chunks, int32_t* offp,
                               int32_t* first, cudaStream_t s) {
  pad_offsets_kernel<<<n_chunks, 32, 0, s>>>(counts, E, offp);
  first_chunk_kernel<<<(E + 127) / 128, 128, 0, s>>>(counts, E, n_chunks, first);
  return cudaGetLastError();
}

cudaError_t launch_zero_pad_rows(const int32_t* off, const int32_t* offp, int32_t E, int32_t H,
                                 void* buf, float* wrow, int64_t rows_cap, cudaStream_t s) {
  static_assert(kPadRows <= 256, "one thread per pad row");
  zero_pad_rows_kernel<<<(unsigned)(E < 1024 ? E : 1024), 256, 0, s>>>(
      off, offp, E, H / 8, static_cast<uint4*>(buf), wrow, rows_cap);
  return cudaGetLastError();
}

cudaError_t launch_pad_rows(const int32_t* idx, const int32_t* dst, const int32_t* off,
                            const int32_t* offp, const float* w, int64_t n, int32_t* dstp,
                            float* wrow, int64_t rows_cap, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  pad_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(idx, dst, off, offp, w, n, dstp,
                                                               wrow, rows_cap);
  return cudaGetLastError();
}

cudaError_t launch_dw_sum(const float* dwp, const int32_t* dstp, int64_t n, int32_t slots,
                          float* dw, int64_t rows_cap, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  dw_sum_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(dwp, dstp, n, slots, dw, rows_cap);
  return cudaGetLastError();
}

cudaError_t launch_sum_rows(const void* dX, const int32_t* dstp, int64_t Tc, int32_t H, int32_t k,
                            void* out, int64_t rows_cap, cudaStream_t s) {
  if (Tc <= 0) return cudaSuccess;
  sum_rows_kernel<<<row_grid(Tc), kRowThreads, 0, s>>>(static_cast<const uint4*>(dX), dstp, Tc,
                                                       H / 8, k, static_cast<uint4*>(out),
                                                       rows_cap);
  return cudaGetLastError();
}

uint32_t checks_take_backward() {
  uint32_t v = 0, zero = 0;
  if (!MOE_CHECKS) return 0;
  cudaMemcpyFromSymbol(&v, g_range_flags, sizeof v);
  cudaMemcpyToSymbol(g_range_flags, &zero, sizeof zero);
  return v;
}

}  // namespace moe
