/*
 * oracle.c -- plain, slow, obviously correct CPU reference of the chunked MoE
 * forward pass.  TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg are its only users.  It shares no code, header,
 * table or helper with the CUDA library and must never be used as a fallback for it.
 *
 * Source of every definition: the MindSpeed article "昇腾MindSpeed分块专家计算Chunk MoE:
 * 让通信藏进计算、显存轻装上阵" ([ChunkMoE] below, cited by section heading).
 *
 * Precision: all floating point work is fp64.  bf16 inputs are widened exactly
 * (bf16 -> fp32 -> fp64).  Nothing is rounded back to bf16: the oracle is the exact
 * function of the bf16-rounded inputs, up to fp64 rounding.
 *
 * Readings of points the article leaves open (each also listed in the design notes):
 *  R1 FFN form: SwiGLU without biases, y = Wd (silu(Wg x) * (Wu x)); W_gate_up[e]
 *     holds gate rows 0..I-1 then up rows I..2I-1.
 *  R2 Order of rows inside one expert: flat index t*k+j ascending (stable).
 *  R3 recv splits on one GPU equal the send splits (one source rank).
 *  R5 An empty chunk or a zero-row expert contributes nothing and is valid.
 *  R6 Duplicate experts in one token's k choices are independent slots; both add.
 *  R7 A chunk size S (with no chunk count) means chunks of exactly S tokens, the last one
 *     holding the remainder.
 *
 * Parity pins: none of these functions is "parity unpinned"; the pins are the
 * property, brute-force, closed-form and golden-fixture tests in tests/.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bits -> fp64, exactly: a bf16 is the top 16 bits of an IEEE fp32. */
static double bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), with the C library's fp64 exp. */
static double silu(double z) { return z / (1.0 + exp(-z)); }

int oracle_effective_chunks(int32_t num_chunks) {
  /* [ChunkMoE] "操作指南" step 3: a chunk setting of 0 means no split, i.e. one chunk. */
  return num_chunks <= 0 ? 1 : num_chunks;
}

/* [ChunkMoE] "一组关键公式": T_chunk = ceil(T / N); chunk c is tokens
 * [c*T_chunk, min(T, (c+1)*T_chunk)).  Writes N_eff + 1 bounds. */
void oracle_chunk_bounds(int64_t T, int32_t num_chunks, int64_t* bounds) {
  int64_t n = oracle_effective_chunks(num_chunks);
  int64_t t_chunk = (T + n - 1) / n; /* ceil(T / N) for T >= 0, N >= 1 */
  for (int64_t c = 0; c <= n; ++c) {
    int64_t b = c * t_chunk;
    bounds[c] = b < T ? b : T;
  }
}

/* Chunking from the two settings of [ChunkMoE] "操作指南" step 3: moe_num_chunks and
 * moe_chunk_size should not both be positive; when both are, moe_num_chunks wins (and a
 * warning is due); when both are 0 the input is not split.  A chunk size S alone means
 * chunks of S tokens, the last one holding the rest (reading R7).  With num_chunks = N the
 * chunk size is T_chunk = ceil(T/N) ("一组关键公式").
 * Writes the chunk count and chunk size; returns 1 if the warning is due, 0 if not, and
 * -1 for a negative setting. */
int oracle_resolve_chunks(int64_t T, int32_t num_chunks, int32_t chunk_size, int32_t* n_out,
                          int64_t* t_chunk_out) {
  if (T < 0 || num_chunks < 0 || chunk_size < 0) return -1;
  if (num_chunks > 0) {
    *n_out = num_chunks;
    *t_chunk_out = (T + num_chunks - 1) / num_chunks;
    return chunk_size > 0;
  }
  if (chunk_size > 0) {
    int64_t n = (T + chunk_size - 1) / chunk_size;
    *n_out = (int32_t)(n > 0 ? n : 1);
    *t_chunk_out = chunk_size;
    return 0;
  }
  *n_out = 1;
  *t_chunk_out = T;
  return 0;
}

/* Chunk bounds for a resolved chunk count n and chunk size: chunk c = tokens
 * [min(T, c*t_chunk), min(T, (c+1)*t_chunk)). */
void oracle_chunk_bounds_sized(int64_t T, int32_t n, int64_t t_chunk, int64_t* bounds) {
  for (int64_t c = 0; c <= n; ++c) {
    int64_t b = c * t_chunk;
    bounds[c] = b < T ? b : T;
  }
}

/* Batched pre-dispatch metadata ([ChunkMoE] "一张专业时序图", batched_pre_dispatch_metadata
 * paragraph: splits to send/receive, per-rank token counts, per-expert token counts for
 * all chunks) and the permutation of [ChunkMoE] "核心原理" (permute groups each token
 * copy by the expert it goes to).
 *
 * By definition, for each chunk c the permuted rows are the chunk's copies (t, j)
 * listed expert by expert (e = 0..E-1), and inside one expert in flat order t*k+j
 * (reading R2).  Row numbers are chunk-local.  Virtual EP group g owns experts
 * [g*E/G, (g+1)*E/G), so listing experts ascending also lists groups ascending.
 *
 * Outputs (N = N_eff): counts [N][E], offsets [N][E+1], send [N][G], recv [N][G],
 * dst [T*k] (chunk-local row of copy t*k+j), src_tok [T*k] (src_tok[bounds[c]*k + r] =
 * token of row r of chunk c).  Any may be NULL.
 * Returns the number of index entries outside [0, E); on a nonzero return the outputs
 * are unspecified.  This enumeration is O(E * T * k): slow on purpose, plainly right. */
int64_t oracle_metadata_sized(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t G,
                              int32_t n, int64_t t_chunk, int32_t* counts, int32_t* offsets,
                              int32_t* send, int32_t* recv, int32_t* dst, int32_t* src_tok) {
  int64_t bad = 0;
  for (int64_t s = 0; s < T * (int64_t)k; ++s)
    if (idx[s] < 0 || idx[s] >= E) ++bad;
  if (bad) return bad;
  if (G <= 0) G = 1;
  int64_t* bounds = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n + 1));
  oracle_chunk_bounds_sized(T, n, t_chunk, bounds);
  int32_t per_group = E / G;
  for (int32_t c = 0; c < n; ++c) {
    int64_t t0 = bounds[c], t1 = bounds[c + 1];
    int32_t row = 0;
    for (int32_t e = 0; e < E; ++e) {
      int32_t start = row;
      for (int64_t t = t0; t < t1; ++t) {
        for (int32_t j = 0; j < k; ++j) {
          if (idx[t * k + j] != e) continue;
          if (dst) dst[t * k + j] = row;
          if (src_tok) src_tok[t0 * k + row] = (int32_t)t;
          ++row;
        }
      }
      if (counts) counts[(int64_t)c * E + e] = row - start;
      if (offsets) offsets[(int64_t)c * (E + 1) + e] = start;
    }
    if (offsets) offsets[(int64_t)c * (E + 1) + E] = row;
    for (int32_t g = 0; g < G; ++g) {
      /* rows bound for group g = rows of its experts, counted directly */
      int32_t rows_g = 0;
      for (int64_t t = t0; t < t1; ++t)
        for (int32_t j = 0; j < k; ++j)
          if (idx[t * k + j] / per_group == g) ++rows_g;
      if (send) send[(int64_t)c * G + g] = rows_g;
      if (recv) recv[(int64_t)c * G + g] = rows_g; /* reading R3: one source rank */
    }
  }
  free(bounds);
  return 0;
}

/* The same with chunks from num_chunks alone (T_chunk = ceil(T/N)). */
int64_t oracle_metadata(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t G,
                        int32_t num_chunks, int32_t* counts, int32_t* offsets, int32_t* send,
                        int32_t* recv, int32_t* dst, int32_t* src_tok) {
  int32_t n = 1;
  int64_t t_chunk = T;
  if (oracle_resolve_chunks(T, num_chunks, 0, &n, &t_chunk) < 0) return -1;
  return oracle_metadata_sized(idx, T, k, E, G, n, t_chunk, counts, offsets, send, recv, dst,
                               src_tok);
}

/* Gate/up half of the SwiGLU expert ([ChunkMoE] "核心原理" expert computation; FFN form
 * by reading R1) for one input row x [H]:  h[i] = silu(g_i) * u_i  with
 * g_i = sum_c Wg[e][i][c] x[c],  u_i = sum_c Wu[e][i][c] x[c]. */
static void gateup_row(const uint16_t* x, const uint16_t* wgu_e, int32_t H, int32_t I,
                       double* h) {
  double* xd = (double*)malloc(sizeof(double) * (size_t)H);
  for (int32_t c = 0; c < H; ++c) xd[c] = bf16_to_f64(x[c]);
  for (int32_t i = 0; i < I; ++i) {
    const uint16_t* wg = wgu_e + (int64_t)i * H;
    const uint16_t* wu = wgu_e + (int64_t)(I + i) * H;
    double g = 0.0, u = 0.0;
    for (int32_t c = 0; c < H; ++c) {
      g += bf16_to_f64(wg[c]) * xd[c];
      u += bf16_to_f64(wu[c]) * xd[c];
    }
    h[i] = silu(g) * u;
  }
  free(xd);
}

/* Down half: y[o] = sum_i Wd[e][o][i] h[i]. */
static void down_row(const double* h, const uint16_t* wd_e, int32_t H, int32_t I, double* y) {
  for (int32_t o = 0; o < H; ++o) {
    const uint16_t* w = wd_e + (int64_t)o * I;
    double acc = 0.0;
    for (int32_t i = 0; i < I; ++i) acc += bf16_to_f64(w[i]) * h[i];
    y[o] = acc;
  }
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* The MoE layer forward, token by token: for each requested token t,
 *   out[t] = sum_{j<k} w[t][j] * FFN_{idx[t][j]}(hidden[t])
 * ([ChunkMoE] "核心原理": every token copy goes to its expert and the results are
 * merged back per token; weighting by top_k_weights per the listed inputs of
 * [ChunkMoE] "一张专业时序图").  Chunking does not appear: the article's chunked
 * pipeline reaches this same unchunked result ("没有谁被省略").
 * tokens: the n_tokens token ids to evaluate (NULL = all T, in order).
 * out: fp64 [n_tokens][H].  Returns the number of out-of-range indices met (those
 * slots are skipped). */
int64_t oracle_forward(const uint16_t* hidden, const int32_t* idx, const float* w,
                       const uint16_t* wgu, const uint16_t* wd, int64_t T, int32_t H, int32_t I,
                       int32_t E, int32_t k, const int64_t* tokens, int64_t n_tokens,
                       double* out, int nthreads) {
  if (!tokens) n_tokens = T;
  set_threads(nthreads);
  int64_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
  for (int64_t n = 0; n < n_tokens; ++n) {
    int64_t t = tokens ? tokens[n] : n;
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    double* acc = out + n * H;
    for (int32_t c = 0; c < H; ++c) acc[c] = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      int32_t e = idx[t * k + j];
      if (e < 0 || e >= E) {
        ++bad;
        continue;
      }
      gateup_row(hidden + t * H, wgu + (int64_t)e * 2 * I * H, H, I, h);
      down_row(h, wd + (int64_t)e * H * I, H, I, y);
      double wt = (double)w[t * k + j];
      for (int32_t c = 0; c < H; ++c) acc[c] += wt * y[c];
    }
    free(h);
    free(y);
  }
  return bad;
}

/* Stage definitions, for checking one kernel at a time. */

/* permute ([ChunkMoE] "核心原理"): X[dst[t*k+j]] = hidden[t], a plain copy of bf16 bits. */
void oracle_permute(const uint16_t* hidden, const int32_t* dst, int64_t Tc, int32_t H, int32_t k,
                    uint16_t* X) {
  for (int64_t t = 0; t < Tc; ++t)
    for (int32_t j = 0; j < k; ++j)
      memcpy(X + (int64_t)dst[t * k + j] * H, hidden + t * H, sizeof(uint16_t) * (size_t)H);
}

/* Gate/up + SwiGLU of each row r of X, with the row's expert from expert_of_row[r]. */
void oracle_gateup_rows(const uint16_t* X, const int32_t* expert_of_row, int64_t rows,
                        const uint16_t* wgu, int32_t H, int32_t I, double* act, int nthreads) {
  set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < rows; ++r)
    gateup_row(X + r * H, wgu + (int64_t)expert_of_row[r] * 2 * I * H, H, I, act + r * I);
}

/* Down projection of each bf16 row r of Act with the row's expert. */
void oracle_down_rows(const uint16_t* act, const int32_t* expert_of_row, int64_t rows,
                      const uint16_t* wd, int32_t H, int32_t I, double* y, int nthreads) {
  set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < rows; ++r) {
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    for (int32_t i = 0; i < I; ++i) h[i] = bf16_to_f64(act[r * I + i]);
    down_row(h, wd + (int64_t)expert_of_row[r] * H * I, H, I, y + r * H);
    free(h);
  }
}

/* Weighted unpermute / combine ([ChunkMoE] "核心原理": unpermute restores token order and
 * merges the k copies; weighted by top_k_weights):
 *   out[t] = sum_{j<k} w[t*k+j] * Y[dst[t*k+j]]   (fp64). */
void oracle_unpermute(const uint16_t* Y, const int32_t* dst, const float* w, int64_t Tc,
                      int32_t H, int32_t k, double* out) {
  for (int64_t t = 0; t < Tc; ++t) {
    double* o = out + t * H;
    for (int32_t c = 0; c < H; ++c) o[c] = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      const uint16_t* y = Y + (int64_t)dst[t * k + j] * H;
      double wt = (double)w[t * k + j];
      for (int32_t c = 0; c < H; ++c) o[c] += wt * bf16_to_f64(y[c]);
    }
  }
}

/* ---- backward ---------------------------------------------------------------------------
 * Gradient of the layer output with respect to its inputs and expert weights.  The article
 * trains through this layer: its backward pass mirrors the forward chunk pipeline through
 * autograd, with the expert computation optionally recomputed (chunk_moe_recompute)
 * ([ChunkMoE] "一张专业时序图", last paragraph of the timing discussion; "一组关键公式" on
 * recompute).  The mathematics is the chain rule through the definition of oracle_forward;
 * for one copy (t, j) with e = idx[t][j], x = hidden[t]:
 *   g = Wg x, u = Wu x, sig = 1/(1+e^-g), h = g sig u, y = Wd h
 *   d_w[t][j] = <dout[t], y>;  dy = w[t][j] dout[t];  dh = Wd^T dy
 *   du = dh * g sig;  dg = dh * u * (sig + g sig (1 - sig))
 *   d_x[t] += Wg^T dg + Wu^T du;  dWd[e] += dy h^T;  dWg[e] += dg x^T;  dWu[e] += du x^T
 * All fp64.  dWgu is [E][2I][H] (gate rows then up rows), dWd is [E][H][I]; both are
 * overwritten.  Returns the number of out-of-range indices (nonzero: outputs unspecified). */
int64_t oracle_backward(const uint16_t* hidden, const int32_t* idx, const float* w,
                        const uint16_t* wgu, const uint16_t* wd, const uint16_t* dout, int64_t T,
                        int32_t H, int32_t I, int32_t E, int32_t k, double* dx, double* dw,
                        double* dWgu, double* dWd, int nthreads) {
  set_threads(nthreads);
  for (int64_t s = 0; s < T * (int64_t)k; ++s)
    if (idx[s] < 0 || idx[s] >= E) return 1;
  memset(dWgu, 0, sizeof(double) * (size_t)E * 2 * I * H);
  memset(dWd, 0, sizeof(double) * (size_t)E * H * I);
  /* per expert (parallel): every copy routed to e, in flat order */
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t e = 0; e < E; ++e) {
    double* x = (double*)malloc(sizeof(double) * (size_t)H);
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* dy = (double*)malloc(sizeof(double) * (size_t)H);
    double* dh = (double*)malloc(sizeof(double) * (size_t)I);
    const uint16_t* wg = wgu + (int64_t)e * 2 * I * H;
    const uint16_t* wu = wg + (int64_t)I * H;
    const uint16_t* wde = wd + (int64_t)e * H * I;
    double* dwg = dWgu + (int64_t)e * 2 * I * H;
    double* dwu = dwg + (int64_t)I * H;
    double* dwd = dWd + (int64_t)e * H * I;
    for (int64_t t = 0; t < T; ++t) {
      for (int32_t j = 0; j < k; ++j) {
        if (idx[t * k + j] != e) continue;
        for (int32_t c = 0; c < H; ++c) x[c] = bf16_to_f64(hidden[t * H + c]);
        for (int32_t i = 0; i < I; ++i) {
          double a = 0.0, b = 0.0;
          for (int32_t c = 0; c < H; ++c) {
            a += bf16_to_f64(wg[(int64_t)i * H + c]) * x[c];
            b += bf16_to_f64(wu[(int64_t)i * H + c]) * x[c];
          }
          g[i] = a;
          u[i] = b;
          h[i] = silu(a) * b;
        }
        double wt = (double)w[t * k + j];
        for (int32_t o = 0; o < H; ++o) dy[o] = wt * bf16_to_f64(dout[t * H + o]);
        for (int32_t i = 0; i < I; ++i) {
          double a = 0.0;
          for (int32_t o = 0; o < H; ++o) a += bf16_to_f64(wde[(int64_t)o * I + i]) * dy[o];
          dh[i] = a;
        }
        for (int32_t o = 0; o < H; ++o)
          for (int32_t i = 0; i < I; ++i) dwd[(int64_t)o * I + i] += dy[o] * h[i];
        for (int32_t i = 0; i < I; ++i) {
          double sig = 1.0 / (1.0 + exp(-g[i]));
          double du = dh[i] * g[i] * sig;
          double dg = dh[i] * u[i] * (sig + g[i] * sig * (1.0 - sig));
          for (int32_t c = 0; c < H; ++c) {
            dwg[(int64_t)i * H + c] += dg * x[c];
            dwu[(int64_t)i * H + c] += du * x[c];
          }
        }
      }
    }
    free(x); free(g); free(u); free(h); free(dy); free(dh);
  }
  /* per token (parallel): d_x and d_w */
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    double* dy = (double*)malloc(sizeof(double) * (size_t)H);
    double* dh = (double*)malloc(sizeof(double) * (size_t)I);
    double* out = dx + t * H;
    for (int32_t c = 0; c < H; ++c) out[c] = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      int32_t e = idx[t * k + j];
      const uint16_t* wg = wgu + (int64_t)e * 2 * I * H;
      const uint16_t* wu = wg + (int64_t)I * H;
      const uint16_t* wde = wd + (int64_t)e * H * I;
      gateup_row(hidden + t * H, wgu + (int64_t)e * 2 * I * H, H, I, h);
      down_row(h, wde, H, I, y);
      double dot = 0.0;
      for (int32_t o = 0; o < H; ++o) dot += bf16_to_f64(dout[t * H + o]) * y[o];
      dw[t * k + j] = dot;
      double wt = (double)w[t * k + j];
      for (int32_t o = 0; o < H; ++o) dy[o] = wt * bf16_to_f64(dout[t * H + o]);
      for (int32_t i = 0; i < I; ++i) {
        double a = 0.0;
        for (int32_t o = 0; o < H; ++o) a += bf16_to_f64(wde[(int64_t)o * I + i]) * dy[o];
        dh[i] = a;
      }
      for (int32_t i = 0; i < I; ++i) {
        double gi = 0.0, ui = 0.0;
        for (int32_t c = 0; c < H; ++c) {
          gi += bf16_to_f64(wg[(int64_t)i * H + c]) * bf16_to_f64(hidden[t * H + c]);
          ui += bf16_to_f64(wu[(int64_t)i * H + c]) * bf16_to_f64(hidden[t * H + c]);
        }
        double sig = 1.0 / (1.0 + exp(-gi));
        double du = dh[i] * gi * sig;
        double dg = dh[i] * ui * (sig + gi * sig * (1.0 - sig));
        for (int32_t c = 0; c < H; ++c)
          out[c] += bf16_to_f64(wg[(int64_t)i * H + c]) * dg + bf16_to_f64(wu[(int64_t)i * H + c]) * du;
      }
    }
    free(h); free(y); free(dy); free(dh);
  }
  return 0;
}
