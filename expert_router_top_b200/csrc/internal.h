// internal.h -- declarations shared by the library's translation units (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ---- metadata (metadata.cu) -----------------------------------------------------------

constexpr int kMetaThreads = 256;       // 8 warps
constexpr int kMetaSlotsPerTile = 2048; // token copies (t, j) handled by one CTA

struct MetaArgs {
  const int32_t* idx;  // [T][k]
  int64_t T;
  int32_t k, E, G, n_chunks;
  int64_t t_chunk;          // ceil(T / n_chunks)
  int32_t tile_tokens;      // tokens per tile (a tile never straddles two chunks)
  int32_t tiles_per_chunk;  // ceil(t_chunk / tile_tokens)
  int32_t* hist;            // [n_chunks * tiles_per_chunk][E] scratch
  int32_t* dst;             // [T*k] chunk-local row of each copy
  int32_t* src_tok;         // [T*k] or nullptr
  int32_t src_relative = 0; // src_tok holds the token's index in its chunk (else in [0, T))
  int32_t* counts;          // [n_chunks][E]
  int32_t* offsets;         // [n_chunks][E+1]
  int32_t* splits;          // [n_chunks][G]
  uint32_t* status;         // device status words: cleared by the kernel, then [0] flags
  int32_t status_words = 1; // words at status to clear
};

inline int32_t meta_tile_tokens(int32_t k) {
  int32_t t = kMetaSlotsPerTile / k;
  return t < 1 ? 1 : t;
}

cudaError_t launch_metadata(const MetaArgs& a, cudaStream_t s);

// ---- permute / unpermute (permute.cu) ----------------------------------------------------

// rows_cap: rows of X (permute) or Y (unpermute); the checks build verifies every dst row
// against it.
// guard (optional): the call's status word; the kernel does nothing when it holds
// MOE_DEV_BAD_INDEX (the metadata of the call found an expert index out of range).
cudaError_t launch_permute(const void* hidden, const int32_t* dst, int64_t Tc, int32_t H,
                           int32_t k, void* X, int64_t rows_cap, cudaStream_t s,
                           const uint32_t* guard = nullptr);
// ctas_per_sm: CTAs of the compile-time-k combine per SM (0: the build's default).  A combine
// that runs beside a grouped GEMM takes fewer, so that every CTA of it is resident next to
// the GEMM's one CTA per SM and all its tokens progress together.
cudaError_t launch_unpermute(const void* Y, const int32_t* dst, const float* w, int64_t Tc,
                             int32_t H, int32_t k, void* out, int64_t rows_cap, cudaStream_t s,
                             int ctas_per_sm = 0, const uint32_t* guard = nullptr);
// Range-violation flags of the checks build, one word per translation unit: read and clear.
uint32_t checks_take_permute();
uint32_t checks_take_gemm();
uint32_t checks_take_backward();
uint32_t checks_take_ep();

// ---- grouped GEMM (gemm.cu) -------------------------------------------------------------

constexpr int kGemmBM = 128;     // rows per tile (one tcgen05.mma M=128 per CTA)
constexpr int kGemmBN = 256;     // MMA N: 128 gate + 128 up columns, or 256 down columns
constexpr int kGemmThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kGatherThreads = 128;  // gathered A: warps 6-9 copy the token rows

struct GemmArgs {
  const void* A;          // [rows][K] bf16 (permuted X, or Act)
  int64_t rows;           // rows in A and in the output
  const void* B;          // weights [E][b_rows][K]
  void* out;              // [rows][out_cols] bf16
  const int32_t* offsets; // dev [E+1]
  int32_t E;
  int32_t K;              // H for gate/up, I for down
  int32_t out_cols;       // I for gate/up, H for down
  int32_t b_rows;         // 2I for gate/up, H for down
  int64_t total_tiles;    // sum over experts of ceil(rows_e / tile rows) * n_tiles; -1: the
                          // kernel counts them from the offsets, one CTA (or pair) per SM,
                          // and does nothing when *status holds MOE_DEV_BAD_INDEX
  uint32_t* status;
  // Gathered A (gate/up only): A row r is row gather[r] of gather_src [gather_src_rows][K]
  // instead of row r of A.  nullptr = plain A.
  const int32_t* gather = nullptr;
  const void* gather_src = nullptr;
  int64_t gather_src_rows = 0;
};

// 2-D bf16 tensor map over a row-major [rows][cols] matrix: boxes of box_rows x 64 columns,
// 128-byte swizzle, zero fill outside the matrix.
bool make_tma_2d_bf16(CUtensorMap* m, const void* base, int64_t rows, int32_t cols,
                      int32_t box_rows);


// 3-D fp32 tensor map over [E][M][N] (row-major per expert) with a 32 x 32 box and the
// 128-byte swizzle: the target of the weight-gradient stores and add-reductions.
bool make_tma_3d_f32(CUtensorMap* m, void* base, int32_t E, int32_t M, int32_t N);
// Whether the down GEMM copies its A rows with the gathering warps (build option).
bool gemm_down_lsu();
// Output tiles of a GEMM launch (tile height per the kernel variant that runs it).
int64_t gemm_total_tiles(const int32_t* counts_host, int32_t E, int32_t out_cols, bool swiglu,
                         bool gather);

cudaError_t launch_grouped_gemm(const GemmArgs& a, bool swiglu, int num_sms, cudaStream_t s,
                                int* err_detail);

// ---- backward (backward.cu) ------------------------------------------------------------

enum BwdGemmMode { kBwdRawGU = 0, kBwdDSwiGLU = 1, kBwdDPlain = 2, kBwdWGrad = 3 };

struct BwdGemmArgs {
  int mode;                    // BwdGemmMode
  const void* A;               // bf16 [A_rows][A_cols]
  int64_t A_rows;
  int32_t A_cols;
  const void* B;               // bf16 [B_rows][B_cols]
  int64_t B_rows;
  int32_t B_cols;
  const int32_t* offsets;      // dev [E+1] padded expert row offsets
  const int32_t* rows_pad_host;  // host [E] padded rows per expert
  int32_t E;
  int32_t M;                   // kBwdWGrad: gradient rows
  int32_t N;                   // output columns
  int32_t K;                   // row-grouped modes: reduction length
  int32_t I;                   // gate/up split of 2I-wide tensors
  int32_t b_rows;              // rows of one expert's weight matrix in B
  void* out0;
  void* out1;
  const void* aux;
  const float* wrow;           // kBwdRawGU, kBwdDSwiGLU: dev [A_rows] routing weight per row
  float* dwp;                  // kBwdDSwiGLU: dev [A_rows][bwd_dw_slots(I)] partial d_w, or null
  float* acc;                  // kBwdWGrad: [E][M][N] fp32 gradient
  const int32_t* first;        // kBwdWGrad: dev [E] first unit (pair of chunks) with rows of
                               // each expert
  int32_t chunk;               // kBwdWGrad: this unit (store where first is this unit, else add)
  uint32_t* status;
};

int bwd_pad_rows();
// Partial inner products per row that the SwiGLU-backward GEMM writes for d_w.
int32_t bwd_dw_slots(int32_t I);
cudaError_t launch_bwd_gemm(const BwdGemmArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_pad_offsets(const int32_t* counts, int32_t E, int32_t n_chunks, int32_t* offp,
                               int32_t* first, cudaStream_t s);
// Zero the pad rows (offp[e] + count_e .. offp[e+1]) of a padded bf16 [rows][H] buffer and,
// where wrow is not null, the same entries of the per-row routing weights.
cudaError_t launch_zero_pad_rows(const int32_t* off, const int32_t* offp, int32_t E, int32_t H,
                                 void* buf, float* wrow, int64_t rows_cap, cudaStream_t s);
// dstp = padded row of each of n copies; wrow[dstp] = w of the copy.
cudaError_t launch_pad_rows(const int32_t* idx, const int32_t* dst, const int32_t* off,
                            const int32_t* offp, const float* w, int64_t n, int32_t* dstp,
                            float* wrow, int64_t rows_cap, cudaStream_t s);
// d_w of each of n copies = the sum of its row's slots partials (fixed order).
cudaError_t launch_dw_sum(const float* dwp, const int32_t* dstp, int64_t n, int32_t slots,
                          float* dw, int64_t rows_cap, cudaStream_t s);
cudaError_t launch_sum_rows(const void* dX, const int32_t* dstp, int64_t Tc, int32_t H, int32_t k,
                            void* out, int64_t rows_cap, cudaStream_t s);

}  // namespace moe
