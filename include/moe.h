/*
 * moe.h -- C ABI of the chunked MoE forward hot path for one NVIDIA B200 (sm_100a).
 *
 * The method is "Chunk MoE" as described in the MindSpeed article
 * "昇腾MindSpeed分块专家计算Chunk MoE: 让通信藏进计算、显存轻装上阵" (cited below
 * as [ChunkMoE] with the article's section heading). One MoE layer's forward
 * pass is split along tokens into N chunks of T_chunk = ceil(T/N) tokens
 * ([ChunkMoE] "一组关键公式"), adjacent chunks run as a pair with a double-buffered
 * expert workspace ([ChunkMoE] "一张专业时序图"), and the split/count metadata of
 * every chunk is computed at once and reaches the host in one device-to-host
 * copy ([ChunkMoE] "一张专业时序图", the paragraph on batched_pre_dispatch_metadata).
 * Per chunk the steps are: permute (dispatch), expert computation, unpermute
 * (combine) ([ChunkMoE] "核心原理").  The article's All-to-All exchanges become a
 * local layout on one GPU: permuted rows are rank-major (virtual EP group
 * ascending) and expert-contiguous, so no collective runs.
 *
 * The expert FFN is SwiGLU without biases:
 *     y = W_down[e] · ( silu(W_gate[e] · x) ⊙ (W_up[e] · x) ),  silu(z) = z / (1 + e^-z)
 * (the article does not state the FFN form; SwiGLU is this library's fixed choice).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - "dev" pointers are CUDA device pointers; "host" pointers are ordinary host memory.
 *  - bf16 tensors are passed as `void*` / `const void*`; each element is an IEEE
 *    bfloat16 (16 bits, row-major).  fp32 is `float`, indices are int32.
 *  - Weights are K-major (the nn.Linear layout):
 *        W_gate_up [E][2I][H]  rows 0..I-1 of expert e are W_gate[e], rows I..2I-1 are W_up[e];
 *        W_down    [E][H][I].
 *  - `stream` is a cudaStream_t passed as `void*` (NULL = legacy default stream).
 *  - Every call returns a moe_status_t and never aborts, traps or exits.  Argument
 *    checks run on the host before anything is launched.  A call that returns an
 *    error other than MOE_ERR_INDEX / MOE_ERR_CUDA has launched nothing.
 *  - The caller owns every buffer, including the workspace.  The library keeps,
 *    per device and created on first use, one extra non-blocking stream, a few
 *    events and one pinned host staging block; nothing else persists between calls.
 *  - Calls are not thread-safe with respect to each other on the same device.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 4

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,         /* null pointer, bad dimension, E % ep_groups != 0, k > E, ... */
  MOE_ERR_INDEX = 2,       /* a top_k_index entry outside [0, E) (detected on the device)  */
  MOE_ERR_ALIGN = 3,       /* a pointer that is not 16-byte aligned                        */
  MOE_ERR_WORKSPACE = 4,   /* ws_bytes smaller than the size the query functions return    */
  MOE_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed                         */
  MOE_ERR_TIMEOUT = 6,     /* a kernel gave up a bounded wait (never expected)             */
  MOE_ERR_UNSUPPORTED = 7  /* shape outside the kernels' limits (see MOE_MAX_*)            */
} moe_status_t;

/* Kernel limits.  Shapes beyond them return MOE_ERR_UNSUPPORTED. */
#define MOE_MAX_EXPERTS 1024   /* E  */
#define MOE_MAX_TOPK 32        /* k  */
#define MOE_MAX_CHUNKS 1048576 /* num_chunks */

/* Shape of one MoE layer call.
 *   T          tokens (rows of hidden / out), T >= 0; T * k < 2^31
 *   H          hidden size, H > 0, H % 8 == 0
 *   I          expert intermediate size, I > 0, I % 8 == 0
 *   E          routed experts, 1 <= E <= MOE_MAX_EXPERTS
 *   k          experts per token, 1 <= k <= min(E, MOE_MAX_TOPK)
 *   ep_groups  G virtual expert-parallel ranks; group g owns experts
 *              [g*E/G, (g+1)*E/G); E % G == 0; 0 is read as 1
 *   num_chunks N >= 0: split into N chunks of T_chunk = ceil(T/N) tokens
 *   chunk_size S >= 0: split into chunks of exactly S tokens (the last holds the rest)
 *              ([ChunkMoE] "操作指南" step 3: set only one of the two; if both are > 0,
 *              num_chunks wins and moe_last_warning() says so; both 0 => no split). */
typedef struct {
  int64_t T;
  int32_t H, I, E, k, ep_groups, num_chunks, chunk_size;
} moe_shape_t;

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(moe_status_t status);

/* MOE_ABI_VERSION of the loaded library. */
MOE_API int32_t moe_abi_version(void);

/* Chunk partition, host arithmetic only ([ChunkMoE] "一组关键公式": T_chunk = ceil(T/N)).
 * Writes N_eff + 1 bounds, N_eff = max(num_chunks, 1): chunk c holds tokens
 * [bounds[c], bounds[c+1]) with bounds[c] = min(T, c * T_chunk).  Trailing chunks may
 * be empty (T=49, N=8 gives seven chunks of 7 and one of 0).
 * Errors: MOE_ERR_ARG if bounds is NULL, T < 0 or num_chunks < 0. */
MOE_API moe_status_t moe_chunk_bounds(int64_t T, int32_t num_chunks, int64_t* bounds /* host [N_eff+1] */);

/* The chunking a shape asks for ([ChunkMoE] "操作指南" step 3): writes the chunk count
 * (>= 1) and the chunk size in tokens.  When both num_chunks and chunk_size are > 0,
 * num_chunks wins and moe_last_warning() returns a warning.  Host arithmetic only.
 * Errors: MOE_ERR_ARG for a NULL argument or a negative setting; MOE_ERR_UNSUPPORTED for
 * more than MOE_MAX_CHUNKS chunks. */
MOE_API moe_status_t moe_resolve_chunks(const moe_shape_t* shape, int32_t* n_chunks,
                                        int64_t* chunk_tokens);

/* The warning of the last call on this host thread that takes a shape (moe_resolve_chunks,
 * moe_workspace_bytes*, moe_metadata_shape, moe_forward*), or "" if it gave none.  The
 * string stays valid until the thread's next such call. */
MOE_API const char* moe_last_warning(void);

/* Device workspace, in bytes, that moe_metadata needs for these sizes; 0 if invalid. */
MOE_API size_t moe_metadata_workspace_bytes(int64_t T, int32_t k, int32_t E, int32_t ep_groups,
                                    int32_t num_chunks);

/* Device workspace, in bytes, that moe_forward needs for this shape; 0 if invalid.
 * It holds the metadata and min(N_eff, 2) expert buffers of T_chunk*k rows, each
 * (H + I) bf16 values per row: the pair double buffer of [ChunkMoE] "一组关键公式"
 * (W_pair = O(2 * T_chunk)).  The permuted input rows and the expert output rows share
 * one buffer, because the down projection runs only after the gate/up projection has
 * consumed every permuted row of the chunk. */
MOE_API size_t moe_workspace_bytes(const moe_shape_t* shape);

/* Batched pre-dispatch metadata for all chunks ([ChunkMoE] "一张专业时序图", the
 * batched_pre_dispatch_metadata paragraph: one pass for all chunks, one host copy).
 *
 * In:  top_k_index  dev int32 [T][k], entries in [0, E)
 * Out (host, caller-allocated, N_eff = max(num_chunks, 1), G = max(ep_groups, 1)):
 *   send_splits   [N_eff][G]   rows of chunk c bound for virtual EP group g
 *   recv_splits   [N_eff][G]   rows group g receives from this rank; on one GPU the
 *                              only source rank is this one, so recv == send
 *   expert_counts [N_eff][E]   rows of chunk c routed to expert e
 *   chunk_bounds  [N_eff + 1]  as moe_chunk_bounds
 * Out (dev, optional: pass NULL to skip):
 *   dst_rows   int32 [T*k]  dst_rows[t*k+j] = chunk-local row of copy (t,j) in the
 *                           permuted layout: experts ascending (hence groups ascending,
 *                           "rank-major"), and inside one expert the flat index t*k+j
 *                           ascending (a stable order).
 *   src_tokens int32 [T*k]  src_tokens[bounds[c]*k + r] = global token t of chunk c's
 *                           permuted row r (the inverse of dst_rows).
 * workspace: dev, >= moe_metadata_workspace_bytes(...), 256-byte aligned.
 * The call blocks the host once (the single metadata copy) and leaves the outputs
 * complete when it returns.
 * Errors: MOE_ERR_ARG, MOE_ERR_ALIGN, MOE_ERR_WORKSPACE, MOE_ERR_UNSUPPORTED (host
 * checks); MOE_ERR_INDEX if any index is outside [0, E) (outputs then unspecified);
 * MOE_ERR_CUDA. */
MOE_API moe_status_t moe_metadata(const int32_t* top_k_index, int64_t T, int32_t k, int32_t E,
                          int32_t ep_groups, int32_t num_chunks, int32_t* send_splits,
                          int32_t* recv_splits, int32_t* expert_counts, int64_t* chunk_bounds,
                          int32_t* dst_rows, int32_t* src_tokens, void* workspace,
                          size_t ws_bytes, void* stream);

/* Size of the fixed device scratch array behind moe_metadata_noalloc (1 MiB). */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)

/* moe_metadata for callers that cannot allocate.  The Chunk MoE pages have no
 * counterpart of this entry point; it exists for callers that must not allocate device
 * or pinned host memory where they need the routing metadata: a runtime whose device
 * memory belongs entirely to its own caching allocator and forbids out-of-band
 * cudaMalloc/cudaFree (cudaFree also synchronizes the whole device), a latency-critical
 * serving path that cannot pay for an allocation, or a plugin that is handed only its
 * inputs and outputs.
 *
 * Same results as moe_metadata, with these differences:
 *  - No workspace argument: the scratch (status word, per-chunk counts, offsets and
 *    splits, per-tile histograms) lives in one file-scope device array of
 *    MOE_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds until the
 *    process exits.  The call needs
 *        a(16 + 4*N*(E+G)) + a(4*N*(E+1)) + a(4*N*ceil(ceil(T/N) / floor(2048/k))*E)
 *    bytes of it (a() rounds up to 256, N = max(num_chunks,1), G = max(ep_groups,1));
 *    larger sizes return MOE_ERR_WORKSPACE before anything is launched.
 *  - dst_rows is required (not NULL) when T > 0; src_tokens stays optional.
 *  - It allocates nothing: no cudaMalloc/cudaFree, no pinned host block, no stream or
 *    event creation; the packed results come back through a fixed host array.
 *  - The first call on each device looks up the device address of the scratch array
 *    (cudaGetSymbolAddress, with that device current); make that first call before any
 *    stream capture.
 *  - Every call shares the one array and finds the previous call's contents in it; the
 *    call clears the status word and overwrites everything else it reads.  Calls whose
 *    work overlaps on the GPU (several streams or host threads) race on the array and
 *    on the host array: serialize them.
 * Errors: as moe_metadata, plus MOE_ERR_WORKSPACE for sizes beyond the array. */
MOE_API moe_status_t moe_metadata_noalloc(const int32_t* top_k_index, int64_t T, int32_t k,
                                          int32_t E, int32_t ep_groups, int32_t num_chunks,
                                          int32_t* send_splits, int32_t* recv_splits,
                                          int32_t* expert_counts, int64_t* chunk_bounds,
                                          int32_t* dst_rows, int32_t* src_tokens, void* stream);

/* moe_metadata with the chunking of a shape (num_chunks or chunk_size, see moe_shape_t;
 * H and I are not used).  The host arrays hold N_eff = the chunk count of
 * moe_resolve_chunks(shape) rows.  workspace: >= moe_workspace_bytes of the same shape (any
 * valid H, I; H = I = 8 gives the smallest size).  Otherwise as moe_metadata. */
MOE_API moe_status_t moe_metadata_shape(const moe_shape_t* shape, const int32_t* top_k_index,
                                        int32_t* send_splits, int32_t* recv_splits,
                                        int32_t* expert_counts, int64_t* chunk_bounds,
                                        int32_t* dst_rows, int32_t* src_tokens, void* workspace,
                                        size_t ws_bytes, void* stream);

/* One MoE layer forward pass, chunked as Chunk MoE ([ChunkMoE] "核心原理",
 * "一张专业时序图", "一组关键公式"):
 *     out[t] = bf16( sum_{j<k} top_k_weights[t][j] * FFN_{top_k_index[t][j]}(hidden[t]) )
 * with the j-sum in fp32 in ascending j.  Steps: metadata for all chunks + one
 * device-to-host copy; then per chunk c: permute, gate/up grouped
 * GEMM with SwiGLU, down grouped GEMM, weighted unpermute.  Chunks run as a two-stream
 * pair pipeline on two workspace buffers: the permute of chunk c+1 and the unpermute of
 * chunk c-1 overlap the expert GEMMs of chunk c.  The result is bit-identical for every
 * num_chunks.
 *
 * In (dev):  hidden [T][H] bf16, top_k_index [T][k] int32, top_k_weights [T][k] fp32,
 *            W_gate_up [E][2I][H] bf16, W_down [E][H][I] bf16
 * Out (dev): out [T][H] bf16, fully overwritten (unspecified after an error; after
 *            MOE_ERR_INDEX not written at all)
 * workspace: dev, >= moe_workspace_bytes(shape), 256-byte aligned; it must not
 *            overlap any input or output.
 * hidden, out, W_gate_up, W_down must be 16-byte aligned; top_k_index and
 * top_k_weights 4-byte aligned.
 * Synchrony: the whole pipeline is enqueued on `stream` (and on the library's second
 * stream, which is joined back into `stream` before the call returns) without waiting for
 * the metadata: the GEMMs count their tiles from the device offsets, and every kernel after
 * the metadata does nothing when it found an expert index out of range.  The host then
 * blocks once, on the metadata copy (done early on the device), to return that status;
 * the caller synchronizes `stream` to read `out`.
 * T == 0 returns MOE_OK and launches nothing.
 * Errors: as moe_metadata.  A kernel that gives up a bounded wait records it in the
 * workspace; moe_check_device_status reports it. */
MOE_API moe_status_t moe_forward(const moe_shape_t* shape, const void* hidden, const int32_t* top_k_index,
                         const float* top_k_weights, const void* W_gate_up, const void* W_down,
                         void* out, void* workspace, size_t ws_bytes, void* stream);

/* Flags of moe_forward_ex. */
#define MOE_FWD_FUSED_DISPATCH 1u    /* gather the gate/up GEMM's rows from hidden; no permute */
#define MOE_FWD_SEPARATE_DISPATCH 2u /* permute kernel first, as the article's permute step */
#define MOE_FWD_PER_CHUNK_GEMMS 4u   /* fused dispatch: one GEMM sweep per chunk, not per pair */

/* moe_forward with a choice of dispatch.  MOE_FWD_SEPARATE_DISPATCH: the permute kernel
 * writes the permuted rows (the article's separate permute step) and the pipeline overlaps
 * the permute of chunk c+1 and the unpermute of chunk c-1 with the expert GEMMs of chunk c.
 * MOE_FWD_FUSED_DISPATCH: the gate/up GEMM copies each permuted row's K blocks straight from
 * `hidden` through the permutation's inverse map (four gathering warps per CTA), so no
 * permuted copy of the input is written or read.  With the fused dispatch the two chunks of
 * each pair (2m, 2m+1) share one tile sweep per GEMM, so each expert's weight tiles are
 * fetched once per pair rather than once per chunk (MOE_FWD_PER_CHUNK_GEMMS: one sweep per
 * chunk), and the unpermutes of pair m overlap the gate/up GEMM of pair m+1.  The routing
 * metadata then runs per pair, so each expert's rows are contiguous over both chunks and a
 * row tile may span them; the workspace is unchanged (the pair's two chunk buffers are
 * resident anyway and hold its rows as one buffer).  flags = 0 (what
 * moe_forward does) chooses fused: it saves the permute kernel and the permuted copy, and
 * with two or more chunks the pair sweeps halve the weight stream.
 * Every choice gives bit-identical outputs; arguments, workspace and errors are as
 * moe_forward (unknown flag bits, or both flags: MOE_ERR_ARG). */
MOE_API moe_status_t moe_forward_ex(const moe_shape_t* shape, const void* hidden,
                                    const int32_t* top_k_index, const float* top_k_weights,
                                    const void* W_gate_up, const void* W_down, void* out,
                                    void* workspace, size_t ws_bytes, uint32_t flags,
                                    void* stream);

/* The dispatch moe_forward_ex takes for this shape and these flags: 1 fused, 0 separate,
 * -1 invalid flags. */
MOE_API int32_t moe_forward_dispatch(const moe_shape_t* shape, uint32_t flags);

/* Device workspace, in bytes, that moe_forward_host needs: the moe_forward workspace plus
 * device staging for the routing arrays (T*k int32 + T*k fp32) and min(N_eff, 2) input
 * and output buffers of T_chunk rows of H bf16.  0 if the shape is invalid. */
MOE_API size_t moe_workspace_bytes_host(const moe_shape_t* shape);

/* moe_forward with the activations in host memory: hidden_host [T][H] bf16,
 * top_k_index_host [T][k] int32, top_k_weights_host [T][k] fp32 and out_host [T][H] bf16
 * are host pointers (pinned memory lets the copies overlap the kernels; pageable memory
 * works but serializes them); the weights stay on the device.  The routing arrays go to
 * the device first (the metadata needs all of them); then chunk c's input rows are copied
 * in while the expert GEMMs of chunk c-1 run, and chunk c's output rows are copied out
 * while the GEMMs of chunk c+1 run, on two library copy streams beside the pair pipeline
 * ([ChunkMoE] "一张专业时序图": transfers hidden behind the neighbouring chunk's compute).
 * Each chunk has its own GEMM sweeps; where one chunk's permuted copy would be a sizeable
 * share of their traffic (4 * T_chunk * k >= E * I), the gate/up GEMM gathers its rows
 * straight from the chunk's staged input rows instead of a permuted copy.
 * The call returns when out_host is complete (it synchronizes `stream`).  Results are
 * bit-identical to moe_forward.  workspace: dev, >= moe_workspace_bytes_host(shape).
 * Errors: as moe_forward. */
MOE_API moe_status_t moe_forward_host(const moe_shape_t* shape, const void* hidden_host,
                                      const int32_t* top_k_index_host,
                                      const float* top_k_weights_host, const void* W_gate_up,
                                      const void* W_down, void* out_host, void* workspace,
                                      size_t ws_bytes, void* stream);

/* Device workspace, in bytes, that moe_backward needs for this shape; 0 if the shape is
 * invalid for it (moe_backward also needs H % 64 == 0 and I % 32 == 0). */
MOE_API size_t moe_backward_workspace_bytes(const moe_shape_t* shape);

/* Backward pass of moe_forward, chunk by chunk, with the expert computation recomputed
 * from `hidden` (the recompute setting of [ChunkMoE] "操作指南"; the backward mirrors the
 * forward chunking, "一张专业时序图").  For the loss sum(out * d_out):
 *   d_hidden [T][H] bf16          gradient of hidden (sum of the k copies' gradients, fp32
 *                                 in ascending j, one rounding)
 *   d_weights [T][k] fp32         d_weights[t][j] = <d_out[t], W_down[e] h(t,j)>
 *   dW_gate_up [E][2I][H] fp32    gradient of W_gate_up (gate rows, then up rows)
 *   dW_down [E][H][I] fp32        gradient of W_down
 * All four outputs are overwritten.  Inputs as moe_forward plus d_out [T][H] bf16.  The
 * intermediate g, u, w h, dY (the d_out row of each copy), dg, du and dX rows are bf16 (fp32
 * accumulation in every GEMM and reduction); d_weights is taken on the I side as
 * <W_down^T d_out[t], h(t,j)> in fp32, so the copies' outputs y are never formed.  Chunks run as the mirrored pair pipeline on the caller's stream and the
 * library's second stream, one unit per pair of chunks (2m, 2m+1): the routing metadata is
 * taken per pair, so each expert's rows are contiguous over both chunks (padded to a
 * multiple of 64 inside the workspace), every GEMM is one tile sweep over the pair's rows,
 * and the weight gradients accumulate per pair in fp32 (the first pair with an expert's
 * rows stores, later pairs add through TMA reductions).  d_hidden and d_weights are
 * bit-identical for every chunking; dW_* are equal up to the fp32 summation order.
 * workspace: dev, >= moe_backward_workspace_bytes(shape): the metadata plus two pair
 * buffers of permuted rows and their routing weights (the next pair is permuted while one
 * computes) and one pair set of the other row buffers (dg | du overwrite the recomputed
 * g | u rows in place) and of the fp32 partials of d_weights.  The
 * host blocks once, on the metadata copy.
 * Errors: as moe_forward; MOE_ERR_ARG also for H % 64 or I % 32 != 0. */
MOE_API moe_status_t moe_backward(const moe_shape_t* shape, const void* hidden,
                                  const int32_t* top_k_index, const float* top_k_weights,
                                  const void* W_gate_up, const void* W_down, const void* d_out,
                                  void* d_hidden, float* d_weights, float* dW_gate_up,
                                  float* dW_down, void* workspace, size_t ws_bytes,
                                  void* stream);

/* Synchronizes `stream` and returns MOE_ERR_TIMEOUT if a kernel of an earlier call that
 * used this workspace gave up a bounded wait, MOE_ERR_INDEX if its last metadata pass
 * saw a bad index, else MOE_OK (or MOE_ERR_CUDA). */
MOE_API moe_status_t moe_check_device_status(const void* workspace, size_t ws_bytes, void* stream);

/* ---- Stage entry points ------------------------------------------------------------
 * The kernels of moe_forward, one call each, on caller buffers.  moe_forward does not
 * call these; they exist so that each step can be run and checked on its own.  None of
 * them synchronizes.  `status` is a dev uint32 word that a kernel ORs with 2 when it
 * gives up a bounded wait (the caller zeroes it beforehand). */

/* Permute / dispatch of one chunk ([ChunkMoE] "核心原理", "一张专业时序图"):
 *   X[dst_rows[t*k+j]] = hidden[t]  for t < Tc, j < k.
 * hidden dev bf16 [Tc][H]; dst_rows dev int32 [Tc*k] (chunk-local rows, a bijection onto
 * [0, Tc*k)); X dev bf16 [Tc*k][H].  hidden and X 16-byte aligned. */
MOE_API moe_status_t moe_permute(const void* hidden, const int32_t* dst_rows, int64_t Tc, int32_t H,
                         int32_t k, void* X, void* stream);

/* Expert gate/up projection with SwiGLU, grouped over experts (the expert computation of
 * [ChunkMoE] "核心原理"): for every row r of expert e (rows offsets[e] .. offsets[e+1]-1)
 *   Act[r] = bf16( silu(X[r] · W_gate[e]^T) ⊙ (X[r] · W_up[e]^T) ), fp32 accumulation.
 * X dev bf16 [rows][H]; expert_offsets dev int32 [E+1] (offsets[0] = 0, nondecreasing,
 * offsets[E] = rows); expert_counts_host host int32 [E] (offsets[e+1] - offsets[e]);
 * W_gate_up dev bf16 [E][2I][H]; Act dev bf16 [rows][I].  16-byte aligned. */
MOE_API moe_status_t moe_grouped_gateup(const void* X, int64_t rows, int32_t H, int32_t I, int32_t E,
                                const int32_t* expert_offsets, const int32_t* expert_counts_host,
                                const void* W_gate_up, void* Act, uint32_t* status, void* stream);

/* Expert down projection, grouped over experts:
 *   Y[r] = bf16( Act[r] · W_down[e]^T ), fp32 accumulation.
 * Act dev bf16 [rows][I]; W_down dev bf16 [E][H][I]; Y dev bf16 [rows][H]; other
 * arguments as moe_grouped_gateup.  Y may alias the X of the gate/up call. */
MOE_API moe_status_t moe_grouped_down(const void* Act, int64_t rows, int32_t H, int32_t I, int32_t E,
                              const int32_t* expert_offsets, const int32_t* expert_counts_host,
                              const void* W_down, void* Y, uint32_t* status, void* stream);

/* Weighted unpermute / combine of one chunk ([ChunkMoE] "核心原理", "一张专业时序图"):
 *   out[t] = bf16( sum_{j<k} w[t*k+j] * float(Y[dst_rows[t*k+j]]) ), fp32, j ascending.
 * Y dev bf16 [Tc*k][H]; dst_rows dev int32 [Tc*k]; w dev fp32 [Tc*k]; out dev bf16
 * [Tc][H].  Y and out 16-byte aligned. */
MOE_API moe_status_t moe_unpermute(const void* Y, const int32_t* dst_rows, const float* top_k_weights,
                           int64_t Tc, int32_t H, int32_t k, void* out, void* stream);

/* ---- Range-checked build ----------------------------------------------------------------
 * libmoe_checks.so is this library compiled with every data-dependent row index (permuted
 * and padded rows, gathered token rows, output rows) compared with the rows of the buffer
 * it addresses before the access; a violation skips the access and raises a flag instead
 * of faulting (it stands in for a memory sanitizer).  moe_checks_enabled: 1 in that build,
 * 0 in libmoe.so.  moe_checks_read synchronizes the device, stores the OR of all flags
 * raised since the last read into *flags (0: every index was in range; always 0 in
 * libmoe.so) and clears them. */
MOE_API int32_t moe_checks_enabled(void);
MOE_API moe_status_t moe_checks_read(uint32_t* flags);

/* ---- Failure-detection self-test -------------------------------------------------------
 * Not part of the Chunk MoE method (the article has no counterpart): it exercises the
 * library's own failure detection.  Launches one kernel whose bounded mbarrier wait has
 * no arrival to wait for; after limit_us microseconds (1 .. 1000000) the wait gives up,
 * sets MOE_DEV_TIMEOUT in *status (dev uint32, overwritten) and the kernel returns, the
 * CUDA context stays usable.  Blocks the host until the kernel ends.  Returns
 * MOE_ERR_TIMEOUT when the timeout was reported (the expected outcome), MOE_OK if the
 * wait completed, MOE_ERR_ARG / MOE_ERR_ALIGN / MOE_ERR_CUDA otherwise. */
MOE_API moe_status_t moe_selftest_wait_timeout(uint32_t* status, uint32_t limit_us, void* stream);

/* ---- Expert parallelism over several GPUs ----------------------------------------------
 * [ChunkMoE] "一张专业时序图" (per chunk: All-to-All dispatch, expert computation, All-to-All
 * combine) and "操作指南" (expert_parallel_size): the E experts are split over W ranks, one
 * GPU each; rank d owns experts [d*E/W, (d+1)*E/W).  Each rank routes its own tokens.  On
 * NVLink/NVSwitch the exchange is fused into the row kernels: moe_ep_dispatch stores every
 * token copy straight into its row of the owning rank's receive buffer (peer stores) and
 * moe_ep_combine reads the expert outputs back from the owning ranks (peer loads) while it
 * forms the weighted sum.  Plain 16-byte loads and stores; no TMA, no multicast.
 *
 * One chunk on every rank, in order:
 *   1. moe_metadata(top_k_index, ..., ep_groups = W, num_chunks, ...) -> expert_counts of
 *      each chunk and dst_rows (the chunk-local, expert-major row of each copy);
 *   2. all-gather the chunk's expert_counts [E] over the ranks -> counts_all [W][E] (the
 *      caller's collective, e.g. torch.distributed);
 *   3. moe_ep_plan -> send_delta [E] (copy it to the device) and recv_offsets [E/W + 1];
 *   4. moe_ep_dispatch into the ranks' receive buffers; then every rank must see all
 *      ranks' dispatches complete (a barrier: a collective on the stream, or the host);
 *   5. moe_grouped_gateup / moe_grouped_down on the receive rows with the local weights
 *      (E/W experts, offsets = recv_offsets), Y written into the receive buffer; barrier;
 *   6. moe_ep_combine -> out rows of the chunk; a barrier before the receive buffer is
 *      reused.
 * Receive layout on rank d: local expert by local expert; inside an expert the source
 * ranks ascending, each source's rows in its own stable (t, j) order.  The results equal
 * moe_forward on all ranks' tokens with all experts, bit for bit (each row meets the same
 * GEMM and the same ascending-j sum).
 * Peer buffers: moe_ipc_handle / moe_ipc_open map another process's device buffer on this
 * GPU (CUDA IPC); the device tables recv_rows / expert_rows hold W such pointers (this
 * rank's own buffer at index rank). */
#define MOE_EP_MAX_RANKS 64
#define MOE_IPC_HANDLE_BYTES 64

/* Host arithmetic.  counts_all [W][E]: expert counts of one chunk on every rank (row s =
 * rank s's expert_counts for the chunk).  Writes, for this rank:
 *   send_delta [E]: the row offset to add to dst_rows of a copy of expert e to get its
 *     row in the receive buffer of rank e / (E/W);
 *   recv_offsets [E/W + 1]: where each local expert's rows start in this rank's receive
 *     buffer, and (last entry) the rows it receives.
 * Errors: MOE_ERR_ARG for NULL pointers, W <= 0, E % W != 0, rank outside [0, W) or a
 * negative count; MOE_ERR_UNSUPPORTED beyond MOE_MAX_EXPERTS / MOE_EP_MAX_RANKS or for
 * offsets beyond int32. */
MOE_API moe_status_t moe_ep_plan(const int32_t* counts_all, int32_t W, int32_t rank, int32_t E,
                                 int32_t* send_delta, int32_t* recv_offsets);

/* recv_rows[e / (E/W)][dst_rows[t*k+j] + send_delta[e]] = hidden[t] for every copy (t, j)
 * of one chunk, e = top_k_index[t*k+j].
 *   hidden [Tc][H] bf16 dev (the chunk's rows, 16-byte aligned); top_k_index, dst_rows
 *   [Tc*k] int32 dev (the chunk's slice, dst_rows chunk-local from moe_metadata with
 *   ep_groups = W); send_delta [E] int32 dev (moe_ep_plan); recv_rows: dev array of W
 *   device pointers, each to a receive buffer of rows_cap rows x H bf16 (peer-mapped).
 * Enqueued on `stream`; returns without waiting.  Entries of top_k_index outside [0, E)
 * are skipped (moe_metadata reports them first).  Errors: MOE_ERR_ARG / MOE_ERR_ALIGN /
 * MOE_ERR_UNSUPPORTED from the host checks, MOE_ERR_CUDA if the launch fails. */
MOE_API moe_status_t moe_ep_dispatch(const void* hidden, const int32_t* top_k_index,
                                     const int32_t* dst_rows, const int32_t* send_delta,
                                     void* const* recv_rows, int64_t Tc, int32_t H, int32_t k,
                                     int32_t E, int32_t W, int64_t rows_cap, void* stream);

/* out[t] = bf16( sum_{j<k} top_k_weights[t*k+j] * expert_rows[r][dst + delta] ), fp32
 * accumulation in ascending j (the arithmetic of moe_unpermute), r = e / (E/W), reading
 * each expert output row from the rank that computed it.  expert_rows: dev array of W
 * device pointers to the ranks' expert-output rows (rows_cap x H bf16, peer-mapped);
 * out [Tc][H] bf16 dev, 16-byte aligned, fully overwritten.  Otherwise as
 * moe_ep_dispatch. */
MOE_API moe_status_t moe_ep_combine(void* const* expert_rows, const int32_t* top_k_index,
                                    const int32_t* dst_rows, const int32_t* send_delta,
                                    const float* top_k_weights, int64_t Tc, int32_t H, int32_t k,
                                    int32_t E, int32_t W, int64_t rows_cap, void* out,
                                    void* stream);

/* CUDA IPC of a caller-owned device buffer (any pointer into a cudaMalloc allocation,
 * e.g. a torch tensor): writes the MOE_IPC_HANDLE_BYTES handle of its allocation and the
 * pointer's offset inside it.  moe_ipc_open, in another process on the same node, maps it
 * and returns the pointer (allocation base + offset); moe_ipc_close unmaps it.  Errors:
 * MOE_ERR_ARG for NULL or a negative offset, MOE_ERR_CUDA if the CUDA call fails (a
 * process cannot open its own handle). */
MOE_API moe_status_t moe_ipc_handle(const void* dev_ptr, void* handle /* host [64] */,
                                    int64_t* offset);
MOE_API moe_status_t moe_ipc_open(const void* handle, int64_t offset, void** dev_ptr);
MOE_API moe_status_t moe_ipc_close(void* dev_ptr, int64_t offset);

/* ---- Kernel timing -----------------------------------------------------------------
 * When enabled, every kernel launch of the calls above is bracketed by two CUDA events
 * recorded on the stream the kernel is launched on.  moe_profile_read synchronizes the
 * device, converts the pending event pairs into per-kind totals and returns them. */
typedef enum {
  MOE_KERNEL_METADATA = 0,  /* the metadata kernels (all passes of one call count as one) */
  MOE_KERNEL_PERMUTE = 1,
  MOE_KERNEL_GATEUP = 2,
  MOE_KERNEL_DOWN = 3,
  MOE_KERNEL_UNPERMUTE = 4,
  /* moe_backward */
  MOE_KERNEL_BWD_GATEUP = 5,   /* recomputed [g u] = X W_gate_up^T with w h = w silu(g) u   */
  MOE_KERNEL_BWD_DSWIGLU = 6,  /* a = dY W_down (dY = d_out rows): SwiGLU backward -> [dg du]
                                  with dh = w a, and the partials of d_w = <a, h>           */
  MOE_KERNEL_BWD_DX = 7,       /* dX = [dg du] W_gate_up                                    */
  MOE_KERNEL_BWD_WGRAD = 8,    /* dW_down += dY^T (w h) and dW_gate_up += [dg du]^T X       */
  MOE_KERNEL_BWD_ROWS = 9,     /* row kernels: padded permute, dY, d_weights sums, d_hidden */
  MOE_KERNEL_KINDS = 10
} moe_kernel_kind_t;

typedef struct {
  int64_t launches[MOE_KERNEL_KINDS];  /* timed launches of each kind                    */
  double ms[MOE_KERNEL_KINDS];         /* summed event-to-event device time, ms           */
  int64_t rows[MOE_KERNEL_KINDS];      /* summed rows processed: tokens for metadata,
                                          permuted rows (T_c*k) for the other kinds        */
  int64_t active_experts[MOE_KERNEL_KINDS]; /* summed experts with >0 rows (GEMM kinds)  */
  int64_t kernels;                     /* device kernels launched while enabled          */
} moe_profile_t;

MOE_API moe_status_t moe_profile_enable(int32_t on);  /* also clears the totals */
MOE_API moe_status_t moe_profile_read(moe_profile_t* out);

/* One timed launch, for a timeline of the two-stream pipeline (the article's section
 * 一张专业时序图 draws Expert(c) beside the dispatch/combine of the neighbouring chunk; these
 * records show which kernels of a call actually ran side by side). */
typedef struct {
  int32_t kind;     /* moe_kernel_kind_t                                                    */
  int32_t stream;   /* 0 the caller's stream, 1 the library's second stream,
                       2 / 3 the copy-in / copy-out streams of moe_forward_host             */
  int64_t call;     /* 1-based index of the library call, since moe_profile_enable, that
                       launched it (moe_forward, moe_forward_host, moe_backward; 0 others)   */
  int64_t rows;     /* as moe_profile_t.rows                                                */
  double start_ms;  /* event times in ms, relative to an event recorded on the first timed
                       launch's stream just before it; events of the other streams may
                       precede it (negative)                                                */
  double end_ms;
} moe_launch_record_t;

/* Synchronizes the device like moe_profile_read, folds the pending launches into the totals
 * and the kept records (the first 65536 since moe_profile_enable), copies up to `capacity`
 * records (host array, caller-owned) in enqueue order and sets *count to the number kept.
 * MOE_ERR_ARG for a null count, a negative capacity or a null array with capacity > 0;
 * MOE_ERR_CUDA if the device or an event query fails. */
MOE_API moe_status_t moe_profile_timeline(moe_launch_record_t* records, int32_t capacity,
                                          int32_t* count);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
