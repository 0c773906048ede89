// moe.cu -- C ABI of the chunked MoE forward pass: argument checks, workspace layout,
// the single metadata copy, and the two-stream pair pipeline over the chunks.
//
// Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE"):
//   一组关键公式  T_chunk = ceil(T/N); the pair double buffer W_pair = O(2 * T_chunk)
//   一张专业时序图 forward_pair over adjacent chunks c and n = c+1: Expert(c) overlaps the
//                 dispatch of n, Expert(n) overlaps the combine of c; the first dispatch and
//                 the last combine stay exposed; batched_pre_dispatch_metadata does one
//                 pass and one host copy for all chunks
//   核心原理      permute -> expert computation -> unpermute per chunk
//   操作指南      a chunk setting of 0 means no split
// On one GPU the article's All-to-All dispatch/combine become the permute/unpermute
// layout itself: rows are expert-contiguous and rank-major, so nothing crosses devices.
//
// Stream roles inside moe_forward: the caller's stream M runs metadata, permute and
// unpermute; the library's stream G runs the two expert GEMMs.  Chunk c uses workspace
// buffer c % 2.  Enqueue order on M is P(0) P(1) U(0) P(2) U(1) ... U(last), so P(c+1)
// runs beside the GEMMs of c and U(c) beside the GEMMs of c+1; P(c+2) follows U(c) on M,
// which frees buffer c % 2 for it.
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "device.cuh"
#include "internal.h"
#include "moe.h"

namespace {

using namespace moe;

#ifndef MOE_UNPERM_BESIDE_GEMM_CTAS_PER_SM
#define MOE_UNPERM_BESIDE_GEMM_CTAS_PER_SM 1  // combine CTAs per SM while a GEMM holds the SMs
#endif

constexpr size_t kAlign = 256;
constexpr int kStatusWords = 4;  // packed block: status words, then counts, then splits
constexpr int kMaxDevices = 64;
constexpr int32_t kMaxChunks = MOE_MAX_CHUNKS;

size_t al(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct Dims {
  int64_t T;
  int32_t k, E, G, n;  // n = effective chunk count
  int64_t t_chunk;
  int32_t tile_tokens, tiles_per_chunk;
};

struct Layout {
  size_t packed, packed_bytes, offsets, hist, dst, src;
  size_t xy[2], act[2];
  int nbuf;
  int64_t rows_cap;
  size_t total;
};

thread_local std::string g_warning;

// [ChunkMoE] "操作指南" step 3: num_chunks wins over chunk_size (with a warning); a chunk
// size alone gives chunks of exactly chunk_size tokens; both 0 means one chunk.
void resolve_chunking(int64_t T, int32_t num_chunks, int32_t chunk_size, int64_t* n,
                      int64_t* t_chunk) {
  if (num_chunks > 0) {
    *n = num_chunks;
    *t_chunk = (T + num_chunks - 1) / num_chunks;
    if (chunk_size > 0)
      g_warning = "moe_num_chunks and moe_chunk_size are both > 0: moe_num_chunks (" +
                  std::to_string(num_chunks) + ") is used, moe_chunk_size (" +
                  std::to_string(chunk_size) + ") is ignored";
  } else if (chunk_size > 0) {
    const int64_t c = (T + chunk_size - 1) / chunk_size;
    *n = c > 0 ? c : 1;
    *t_chunk = chunk_size;
  } else {
    *n = 1;
    *t_chunk = T;
  }
}

Dims make_dims(int64_t T, int32_t k, int32_t E, int32_t ep_groups, int32_t num_chunks,
               int32_t chunk_size = 0) {
  Dims d;
  d.T = T;
  d.k = k;
  d.E = E;
  d.G = ep_groups > 0 ? ep_groups : 1;
  int64_t n = 1, tc = T;
  resolve_chunking(T, num_chunks, chunk_size, &n, &tc);
  d.n = (int32_t)n;
  d.t_chunk = tc < T ? tc : T;  // a chunk size above T still means one chunk of T tokens
  d.tile_tokens = meta_tile_tokens(k);
  d.tiles_per_chunk = (int32_t)((d.t_chunk + d.tile_tokens - 1) / d.tile_tokens);
  if (d.tiles_per_chunk < 1) d.tiles_per_chunk = 1;
  return d;
}

// The pairs of chunks (2m, 2m+1) as chunks of their own: ceil(n/2) chunks of 2 t_chunk
// tokens, pair m covering exactly the tokens of its two chunks.  Routing metadata at this
// granularity lays the rows of each expert out contiguously over both chunks of a pair, so
// one GEMM sweep serves the pair with row tiles that may span its two chunks.
Dims pair_dims(const Dims& d) {
  Dims p = d;
  p.n = (d.n + 1) / 2;
  p.t_chunk = 2 * d.t_chunk < d.T ? 2 * d.t_chunk : d.T;
  p.tiles_per_chunk = (int32_t)((p.t_chunk + p.tile_tokens - 1) / p.tile_tokens);
  if (p.tiles_per_chunk < 1) p.tiles_per_chunk = 1;
  return p;
}

// Workspace layout.  with_buffers: the expert buffers of moe_forward (whose metadata may run
// per chunk or per pair of chunks); with_dst/with_src: scratch for the permutation when the
// caller does not provide it.
Layout make_layout(const Dims& d, int32_t H, int32_t I, bool with_buffers, bool with_dst,
                   bool with_src) {
  Layout L{};
  size_t o = 0;
  L.packed = o;
  L.packed_bytes = sizeof(int32_t) * (kStatusWords + (size_t)d.n * d.E + (size_t)d.n * d.G);
  o += al(L.packed_bytes);
  L.offsets = o;
  o += al(sizeof(int32_t) * (size_t)d.n * (d.E + 1));
  L.hist = o;
  size_t hist_tiles = (size_t)d.n * d.tiles_per_chunk;
  if (with_buffers) {
    const Dims p = pair_dims(d);
    if ((size_t)p.n * p.tiles_per_chunk > hist_tiles) hist_tiles = (size_t)p.n * p.tiles_per_chunk;
  }
  o += al(sizeof(int32_t) * hist_tiles * d.E);
  L.dst = o;
  if (with_dst) o += al(sizeof(int32_t) * (size_t)(d.T * d.k));
  L.src = o;
  if (with_src) o += al(sizeof(int32_t) * (size_t)(d.T * d.k));
  L.nbuf = 0;
  L.rows_cap = d.t_chunk * d.k;
  if (with_buffers) {
    // the pair double buffer: one buffer for N = 1, two otherwise.  The two X|Y buffers are
    // adjacent, and so are the two Act buffers: a pair's rows fill both as one buffer.
    L.nbuf = d.n >= 2 ? 2 : 1;
    for (int b = 0; b < L.nbuf; ++b) {
      L.xy[b] = o;
      o += al(sizeof(uint16_t) * (size_t)L.rows_cap * H);
    }
    for (int b = 0; b < L.nbuf; ++b) {
      L.act[b] = o;
      o += al(sizeof(uint16_t) * (size_t)L.rows_cap * I);
    }
  }
  L.total = o;
  return L;
}

// Extra device staging of moe_forward_host, placed after the moe_forward layout.
struct HostStaging {
  size_t idx, w, in[2], out[2], total;
};

HostStaging make_host_staging(const Dims& d, int32_t H, size_t base) {
  HostStaging h{};
  size_t o = base;
  h.idx = o;
  o += al(sizeof(int32_t) * (size_t)(d.T * d.k));
  h.w = o;
  o += al(sizeof(float) * (size_t)(d.T * d.k));
  const int nbuf = d.n >= 2 ? 2 : 1;
  for (int b = 0; b < 2; ++b) {
    if (b < nbuf) {
      h.in[b] = o;
      o += al(sizeof(uint16_t) * (size_t)d.t_chunk * H);
      h.out[b] = o;
      o += al(sizeof(uint16_t) * (size_t)d.t_chunk * H);
    } else {
      h.in[b] = h.in[0];
      h.out[b] = h.out[0];
    }
  }
  h.total = o;
  return h;
}

std::vector<int64_t> dims_bounds(const Dims& d) {
  std::vector<int64_t> b((size_t)d.n + 1);
  for (int64_t c = 0; c <= d.n; ++c) b[c] = c * d.t_chunk < d.T ? c * d.t_chunk : d.T;
  return b;
}

moe_status_t check_routing_dims(int64_t T, int32_t k, int32_t E, int32_t ep_groups,
                                int32_t num_chunks) {
  if (T < 0 || k <= 0 || E <= 0 || ep_groups < 0 || num_chunks < 0) return MOE_ERR_ARG;
  const int32_t G = ep_groups > 0 ? ep_groups : 1;
  if (k > E || E % G != 0) return MOE_ERR_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK || num_chunks > kMaxChunks) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_shape(const moe_shape_t* s) {
  g_warning.clear();
  if (!s) return MOE_ERR_ARG;
  moe_status_t st = check_routing_dims(s->T, s->k, s->E, s->ep_groups, s->num_chunks);
  if (st != MOE_OK) return st;
  if (s->chunk_size < 0) return MOE_ERR_ARG;
  int64_t n = 1, tc = 0;
  resolve_chunking(s->T, s->num_chunks, s->chunk_size, &n, &tc);
  if (n > kMaxChunks) return MOE_ERR_UNSUPPORTED;
  if (s->H <= 0 || s->I <= 0 || s->H % 8 != 0 || s->I % 8 != 0) return MOE_ERR_ARG;
  return MOE_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---- per-device context -------------------------------------------------------------------

struct DeviceCtx {
  bool ready = false;
  int num_sms = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_start = nullptr, ev_join = nullptr, ev_perm[2] = {}, ev_gemm[2] = {},
              ev_unperm[2] = {}, ev_packed = nullptr;
  // host-buffer forward: copy-in / copy-out streams and their events
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t ev_in[2] = {}, ev_in_free[2] = {}, ev_out[2] = {}, ev_out_free[2] = {},
              ev_copy_join = nullptr;
  // backward pipeline, one unit per pair of chunks: permuted rows ready (per X buffer),
  // recomputed Y ready / weight gradients done, dY scattered / d_weights read Y, dX ready,
  // d_hidden rows summed, a unit's weight gradients done with its X buffer (per X buffer)
  cudaEvent_t ev_bp[2] = {}, ev_bf[2] = {}, ev_bdy[2] = {}, ev_bdx[1] = {}, ev_bsum[1] = {},
              ev_bw[2] = {};
  int32_t* host_stage = nullptr;
  size_t host_stage_bytes = 0;
};

DeviceCtx g_ctx[kMaxDevices];
std::mutex g_mu;

moe_status_t get_ctx(DeviceCtx** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceCtx& c = g_ctx[dev];
  if (!c.ready) {
    if (cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&c.side, cudaStreamNonBlocking) != cudaSuccess)
      return MOE_ERR_CUDA;
    const unsigned fl = cudaEventDisableTiming;
    if (cudaEventCreateWithFlags(&c.ev_start, fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_join, fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_perm[0], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_perm[1], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_gemm[0], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_gemm[1], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_unperm[0], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_unperm[1], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_packed, cudaEventDisableTiming) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&c.copy_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c.copy_out, cudaStreamNonBlocking) != cudaSuccess)
      return MOE_ERR_CUDA;
    for (int b = 0; b < 2; ++b)
      if (cudaEventCreateWithFlags(&c.ev_in[b], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.ev_in_free[b], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.ev_out[b], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.ev_out_free[b], fl) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaEventCreateWithFlags(&c.ev_copy_join, fl) != cudaSuccess) return MOE_ERR_CUDA;
    for (int b = 0; b < 2; ++b)
      if (cudaEventCreateWithFlags(&c.ev_bp[b], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.ev_bw[b], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.ev_bf[b], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&c.ev_bdy[b], fl) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaEventCreateWithFlags(&c.ev_bdx[0], fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.ev_bsum[0], fl) != cudaSuccess)
      return MOE_ERR_CUDA;
    c.ready = true;
  }
  *out = &c;
  return MOE_OK;
}

moe_status_t ensure_host_stage(DeviceCtx* c, size_t bytes) {
  if (c->host_stage_bytes >= bytes) return MOE_OK;
  if (c->host_stage) cudaFreeHost(c->host_stage);
  c->host_stage = nullptr;
  c->host_stage_bytes = 0;
  size_t want = bytes < 65536 ? 65536 : bytes;
  void* p = nullptr;
  if (cudaMallocHost(&p, want) != cudaSuccess) return MOE_ERR_CUDA;
  c->host_stage = static_cast<int32_t*>(p);
  c->host_stage_bytes = want;
  return MOE_OK;
}

// ---- kernel timing ------------------------------------------------------------------------

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  int64_t rows, active;
  int kernels;
  int stream_id;  // 0 the caller's stream, 1 the library's side stream, 2 copy-in, 3 copy-out
  int64_t call;   // library call (since moe_profile_enable) that launched the kernel
};

constexpr size_t kTimelineCap = 65536;  // launch records kept for moe_profile_timeline

struct Prof {
  bool on = false;
  std::vector<ProfRec> pending;
  std::vector<cudaEvent_t> pool;
  moe_profile_t tot{};
  cudaEvent_t origin = nullptr;  // recorded before the first timed launch since enable
  bool origin_set = false;
  int64_t calls = 0;
  std::vector<moe_launch_record_t> timeline;
  // GEMM launches enqueued before the host had the call's counts: (pending index, counts
  // row) whose active-expert count is filled in once the counts arrive
  std::vector<std::pair<size_t, int>> fix_active;
} g_prof;

cudaEvent_t prof_event() {
  if (!g_prof.pool.empty()) {
    cudaEvent_t e = g_prof.pool.back();
    g_prof.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

int prof_stream_id(cudaStream_t s) {
  for (const DeviceCtx& c : g_ctx) {
    if (!c.ready) continue;
    if (s == c.side) return 1;
    if (s == c.copy_in) return 2;
    if (s == c.copy_out) return 3;
  }
  return 0;
}

// One library call: numbers the launch records of the call (for the timeline).
struct ProfCall {
  ProfCall() {
    if (g_prof.on) ++g_prof.calls;
    g_prof.fix_active.clear();  // left by a call that returned early
  }
};

struct ProfScope {
  bool on;
  ProfRec r;
  cudaStream_t s;
  int fix_row = -1;  // >= 0: r.active comes later from this row of the call's counts
  ProfScope(int kind, cudaStream_t st, int64_t rows, int64_t active, int kernels)
      : on(g_prof.on), s(st) {
    if (!on) return;
    r.kind = kind;
    r.rows = rows;
    r.active = active;
    r.kernels = kernels;
    r.stream_id = prof_stream_id(st);
    r.call = g_prof.calls;
    if (!g_prof.origin_set) {
      if (!g_prof.origin) g_prof.origin = prof_event();
      cudaEventRecord(g_prof.origin, s);
      g_prof.origin_set = true;
    }
    r.a = prof_event();
    r.b = prof_event();
    cudaEventRecord(r.a, s);
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(r.b, s);
    if (fix_row >= 0) g_prof.fix_active.push_back({g_prof.pending.size(), fix_row});
    g_prof.pending.push_back(r);
  }
};

// The active-expert counts of the launches enqueued before the counts reached the host.
void prof_fix_active(const int32_t* counts, int32_t E) {
  for (const auto& f : g_prof.fix_active) {
    if (f.first >= g_prof.pending.size()) continue;
    int64_t a = 0;
    for (int32_t e = 0; e < E; ++e) a += counts[(size_t)f.second * E + e] > 0;
    g_prof.pending[f.first].active = a;
  }
  g_prof.fix_active.clear();
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// NVTX range on the host timeline around the enqueue of one call, pair or chunk (a profiler
// such as Nsight Systems shows it beside the kernels it launched; without one attached the
// push and pop are no-ops).
struct NvtxRange {
  explicit NvtxRange(const char* fmt, int a = 0, int b = 0) {
    char buf[96];
    snprintf(buf, sizeof buf, fmt, a, b);
    nvtxRangePushA(buf);
  }
  ~NvtxRange() { nvtxRangePop(); }
};

moe_status_t run_metadata(const Dims& d, const int32_t* idx, uint8_t* ws, const Layout& L,
                          int32_t* dst, int32_t* src, cudaStream_t s, bool src_relative = false) {
  MetaArgs a;
  a.src_relative = src_relative ? 1 : 0;
  a.idx = idx;
  a.T = d.T;
  a.k = d.k;
  a.E = d.E;
  a.G = d.G;
  a.n_chunks = d.n;
  a.t_chunk = d.t_chunk;
  a.tile_tokens = d.tile_tokens;
  a.tiles_per_chunk = d.tiles_per_chunk;
  a.hist = reinterpret_cast<int32_t*>(ws + L.hist);
  a.dst = dst;
  a.src_tok = src;
  int32_t* packed = reinterpret_cast<int32_t*>(ws + L.packed);
  a.status = reinterpret_cast<uint32_t*>(packed);
  a.counts = packed + kStatusWords;
  a.splits = a.counts + (size_t)d.n * d.E;
  a.offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  a.status_words = kStatusWords;  // cleared by the kernel
  {
    ProfScope ps(MOE_KERNEL_METADATA, s, d.T, 0, 1);
    if (launch_metadata(a, s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// The single device-to-host copy of {status, counts, splits} for every chunk, enqueued on s
// without waiting for it (fetch_packed_wait does).
moe_status_t fetch_packed_async(DeviceCtx* c, const uint8_t* ws, const Layout& L,
                                cudaStream_t s) {
  moe_status_t st = ensure_host_stage(c, L.packed_bytes);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(c->host_stage, ws + L.packed, L.packed_bytes, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaEventRecord(c->ev_packed, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t fetch_packed_wait(DeviceCtx* c) {
  if (cudaEventSynchronize(c->ev_packed) != cudaSuccess) return MOE_ERR_CUDA;
  const uint32_t status = static_cast<uint32_t>(c->host_stage[0]);
  if (status & MOE_DEV_BAD_INDEX) return MOE_ERR_INDEX;
  if (status & MOE_DEV_TIMEOUT) return MOE_ERR_TIMEOUT;
  return MOE_OK;
}

// The single device-to-host copy of {status, counts, splits} for every chunk.
moe_status_t fetch_packed(DeviceCtx* c, const uint8_t* ws, const Layout& L, cudaStream_t s) {
  moe_status_t st = ensure_host_stage(c, L.packed_bytes);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(c->host_stage, ws + L.packed, L.packed_bytes, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  const uint32_t status = static_cast<uint32_t>(c->host_stage[0]);
  if (status & MOE_DEV_BAD_INDEX) return MOE_ERR_INDEX;
  if (status & MOE_DEV_TIMEOUT) return MOE_ERR_TIMEOUT;
  return MOE_OK;
}

int64_t active_experts(const int32_t* counts, int32_t E) {
  int64_t a = 0;
  for (int32_t e = 0; e < E; ++e) a += counts[e] > 0;
  return a;
}


moe_status_t gemm_call(const void* A, int64_t rows, const void* B, void* out,
                       const int32_t* offsets_dev, const int32_t* counts_host, int32_t E,
                       int32_t K, int32_t out_cols, int32_t b_rows, bool swiglu,
                       uint32_t* status, int num_sms, cudaStream_t s,
                       const int32_t* gather = nullptr, const void* gather_src = nullptr,
                       int64_t gather_src_rows = 0, int fix_row = -1) {
  // counts_host == nullptr: the host has not seen the counts yet; the kernel counts its tiles
  // from the device offsets (and the profile's active-expert count waits for row fix_row)
  GemmArgs g;
  const int64_t active = counts_host ? active_experts(counts_host, E) : 0;
  if (!swiglu && !gather_src && gemm_down_lsu()) {
    gather_src = A;  // the A rows themselves, copied by the gathering warps
    gather_src_rows = rows;
  }
  g.gather = gather;
  g.gather_src = gather_src;
  g.gather_src_rows = gather_src_rows;
  g.A = A;
  g.rows = rows;
  g.B = B;
  g.out = out;
  g.offsets = offsets_dev;
  g.E = E;
  g.K = K;
  g.out_cols = out_cols;
  g.b_rows = b_rows;
  g.total_tiles =
      counts_host ? gemm_total_tiles(counts_host, E, out_cols, swiglu, gather_src != nullptr)
                  : -1;
  g.status = status;
  if (g.total_tiles == 0 || rows == 0) return MOE_OK;
  int detail = 0;
  ProfScope ps(swiglu ? MOE_KERNEL_GATEUP : MOE_KERNEL_DOWN, s, rows, active, 1);
  if (!counts_host) ps.fix_row = fix_row;
  cudaError_t e = launch_grouped_gemm(g, swiglu, num_sms, s, &detail);
  if (e != cudaSuccess) return detail == 1 ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

// ========================================================================================
// C ABI
// ========================================================================================

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_ARG: return "MOE_ERR_ARG: invalid argument";
    case MOE_ERR_INDEX: return "MOE_ERR_INDEX: top_k_index entry outside [0, E)";
    case MOE_ERR_ALIGN: return "MOE_ERR_ALIGN: pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside kernel limits";
  }
  return "unknown moe_status_t";
}

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status_t moe_chunk_bounds(int64_t T, int32_t num_chunks, int64_t* bounds) {
  if (!bounds || T < 0 || num_chunks < 0) return MOE_ERR_ARG;
  const int64_t n = num_chunks > 0 ? num_chunks : 1;
  const int64_t tc = (T + n - 1) / n;
  for (int64_t c = 0; c <= n; ++c) bounds[c] = c * tc < T ? c * tc : T;
  return MOE_OK;
}

size_t moe_metadata_workspace_bytes(int64_t T, int32_t k, int32_t E, int32_t ep_groups,
                                    int32_t num_chunks) {
  if (check_routing_dims(T, k, E, ep_groups, num_chunks) != MOE_OK) return 0;
  return make_layout(make_dims(T, k, E, ep_groups, num_chunks), 8, 8, false, true, true).total;
}

size_t moe_workspace_bytes(const moe_shape_t* s) {
  if (check_shape(s) != MOE_OK) return 0;
  return make_layout(make_dims(s->T, s->k, s->E, s->ep_groups, s->num_chunks, s->chunk_size),
                     s->H, s->I, true, true, true)
      .total;
}

moe_status_t moe_resolve_chunks(const moe_shape_t* shape, int32_t* n_chunks,
                                int64_t* chunk_tokens) {
  g_warning.clear();
  if (!shape || !n_chunks || !chunk_tokens) return MOE_ERR_ARG;
  if (shape->T < 0 || shape->num_chunks < 0 || shape->chunk_size < 0) return MOE_ERR_ARG;
  int64_t n = 1, tc = 0;
  resolve_chunking(shape->T, shape->num_chunks, shape->chunk_size, &n, &tc);
  if (n > kMaxChunks) return MOE_ERR_UNSUPPORTED;
  *n_chunks = (int32_t)n;
  *chunk_tokens = tc;
  return MOE_OK;
}

const char* moe_last_warning(void) { return g_warning.c_str(); }

static moe_status_t metadata_impl(const Dims& d, const int32_t* top_k_index, int32_t* send_splits,
                                  int32_t* recv_splits, int32_t* expert_counts,
                                  int64_t* chunk_bounds, int32_t* dst_rows, int32_t* src_tokens,
                                  void* workspace, size_t ws_bytes, void* stream) {
  if (!send_splits || !recv_splits || !expert_counts || !chunk_bounds) return MOE_ERR_ARG;
  if (d.T > 0 && (!top_k_index || !workspace)) return MOE_ERR_ARG;
  if (!aligned(top_k_index, 4) || !aligned(dst_rows, 4) || !aligned(src_tokens, 4) ||
      !aligned(workspace, kAlign))
    return MOE_ERR_ALIGN;
  const std::vector<int64_t> bounds = dims_bounds(d);
  memcpy(chunk_bounds, bounds.data(), sizeof(int64_t) * bounds.size());
  if (d.T == 0) {
    memset(send_splits, 0, sizeof(int32_t) * (size_t)d.n * d.G);
    memset(recv_splits, 0, sizeof(int32_t) * (size_t)d.n * d.G);
    memset(expert_counts, 0, sizeof(int32_t) * (size_t)d.n * d.E);
    return MOE_OK;
  }
  const Layout L = make_layout(d, 8, 8, false, dst_rows == nullptr, false);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceCtx* ctx = nullptr;
  moe_status_t st = get_ctx(&ctx);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* dst = dst_rows ? dst_rows : reinterpret_cast<int32_t*>(ws + L.dst);
  if ((st = run_metadata(d, top_k_index, ws, L, dst, src_tokens, s)) != MOE_OK) return st;
  if ((st = fetch_packed(ctx, ws, L, s)) != MOE_OK) return st;
  const int32_t* counts = ctx->host_stage + kStatusWords;
  const int32_t* splits = counts + (size_t)d.n * d.E;
  memcpy(expert_counts, counts, sizeof(int32_t) * (size_t)d.n * d.E);
  memcpy(send_splits, splits, sizeof(int32_t) * (size_t)d.n * d.G);
  memcpy(recv_splits, splits, sizeof(int32_t) * (size_t)d.n * d.G);  // one source rank
  return MOE_OK;
}

moe_status_t moe_metadata(const int32_t* top_k_index, int64_t T, int32_t k, int32_t E,
                          int32_t ep_groups, int32_t num_chunks, int32_t* send_splits,
                          int32_t* recv_splits, int32_t* expert_counts, int64_t* chunk_bounds,
                          int32_t* dst_rows, int32_t* src_tokens, void* workspace,
                          size_t ws_bytes, void* stream) {
  moe_status_t st = check_routing_dims(T, k, E, ep_groups, num_chunks);
  if (st != MOE_OK) return st;
  return metadata_impl(make_dims(T, k, E, ep_groups, num_chunks), top_k_index, send_splits,
                       recv_splits, expert_counts, chunk_bounds, dst_rows, src_tokens,
                       workspace, ws_bytes, stream);
}

moe_status_t moe_metadata_shape(const moe_shape_t* shape, const int32_t* top_k_index,
                                int32_t* send_splits, int32_t* recv_splits,
                                int32_t* expert_counts, int64_t* chunk_bounds, int32_t* dst_rows,
                                int32_t* src_tokens, void* workspace, size_t ws_bytes,
                                void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  return metadata_impl(make_dims(shape->T, shape->k, shape->E, shape->ep_groups,
                                 shape->num_chunks, shape->chunk_size),
                       top_k_index, send_splits, recv_splits, expert_counts, chunk_bounds,
                       dst_rows, src_tokens, workspace, ws_bytes, stream);
}

int32_t moe_forward_dispatch(const moe_shape_t* shape, uint32_t flags) {
  const uint32_t both = MOE_FWD_FUSED_DISPATCH | MOE_FWD_SEPARATE_DISPATCH;
  if ((flags & ~(both | MOE_FWD_PER_CHUNK_GEMMS)) || (flags & both) == both || !shape) return -1;
  if (flags & MOE_FWD_SEPARATE_DISPATCH) return 0;
  if (flags & MOE_FWD_FUSED_DISPATCH) return 1;
  if (check_shape(shape) != MOE_OK) return 0;
  // the gathered rows (their copies arriving on the ring by themselves) cost the gate/up
  // GEMM less than the permute kernel and its permuted copy cost the step, at every measured
  // shape and chunk count; with two or more chunks the pair sweeps also halve the weight
  // stream
  return 1;
}

moe_status_t moe_forward(const moe_shape_t* shape, const void* hidden, const int32_t* top_k_index,
                         const float* top_k_weights, const void* W_gate_up, const void* W_down,
                         void* out, void* workspace, size_t ws_bytes, void* stream) {
  return moe_forward_ex(shape, hidden, top_k_index, top_k_weights, W_gate_up, W_down, out,
                        workspace, ws_bytes, 0u, stream);
}

moe_status_t moe_forward_ex(const moe_shape_t* shape, const void* hidden,
                            const int32_t* top_k_index, const float* top_k_weights,
                            const void* W_gate_up, const void* W_down, void* out,
                            void* workspace, size_t ws_bytes, uint32_t flags, void* stream) {
  NvtxRange range("moe_forward");
  ProfCall prof_call;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  const int32_t choice = moe_forward_dispatch(shape, flags);
  if (choice < 0) return MOE_ERR_ARG;
  const int64_t T = shape->T;
  const int32_t H = shape->H, I = shape->I, E = shape->E, k = shape->k;
  if (T == 0) return MOE_OK;
  const bool fused = choice == 1;
  // fused dispatch: one GEMM sweep per pair of chunks unless asked for per-chunk GEMMs
  const bool pair_gemms = fused && !(flags & MOE_FWD_PER_CHUNK_GEMMS);
  if (!hidden || !top_k_index || !top_k_weights || !W_gate_up || !W_down || !out || !workspace)
    return MOE_ERR_ARG;
  if (!aligned(hidden, 16) || !aligned(out, 16) || !aligned(W_gate_up, 16) ||
      !aligned(W_down, 16) || !aligned(top_k_index, 4) || !aligned(top_k_weights, 4) ||
      !aligned(workspace, kAlign))
    return MOE_ERR_ALIGN;
  const Dims d = make_dims(T, k, E, shape->ep_groups, shape->num_chunks, shape->chunk_size);
  const Layout L = make_layout(d, H, I, true, true, true);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  DeviceCtx* ctx = nullptr;
  if ((st = get_ctx(&ctx)) != MOE_OK) return st;
  cudaStream_t sm = static_cast<cudaStream_t>(stream);
  cudaStream_t sg = ctx->side;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* dst = reinterpret_cast<int32_t*>(ws + L.dst);
  int32_t* src = reinterpret_cast<int32_t*>(ws + L.src);
  uint32_t* dev_status = reinterpret_cast<uint32_t*>(ws + L.packed);

  // 1) metadata for all chunks (with pair sweeps: for all pairs, so that each expert's rows
  // are contiguous over both chunks of a pair), 2) the one device-to-host copy, on the side
  // stream so that the next launch on this stream need not wait for it, and which the host
  // waits for only after it has enqueued the whole pipeline: nothing below needs the counts
  // on the host (each GEMM counts its tiles from the device offsets), and every kernel does
  // nothing when the metadata flagged an expert index out of range, in which case the call
  // returns MOE_ERR_INDEX as before
  const Dims dm = pair_gemms ? pair_dims(d) : d;
  if ((st = run_metadata(dm, top_k_index, ws, L, dst, src, sm)) != MOE_OK) return st;
  if (cudaEventRecord(ctx->ev_start, sm) != cudaSuccess ||
      cudaStreamWaitEvent(sg, ctx->ev_start, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  if ((st = fetch_packed_async(ctx, ws, L, sg)) != MOE_OK) return st;
  std::vector<int64_t> bounds = dims_bounds(d);
  int n_live = 0;  // chunks with tokens; only trailing chunks can be empty
  while (n_live < d.n && bounds[n_live + 1] > bounds[n_live]) ++n_live;

  const uint16_t* hid = static_cast<const uint16_t*>(hidden);
  uint16_t* outp = static_cast<uint16_t*>(out);
  auto xy = [&](int c) { return ws + L.xy[c % L.nbuf]; };
  auto act = [&](int c) { return ws + L.act[c % L.nbuf]; };
  auto len = [&](int c) { return bounds[c + 1] - bounds[c]; };

  auto permute = [&](int c) -> moe_status_t {
    ProfScope ps(MOE_KERNEL_PERMUTE, sm, len(c) * k, 0, 1);
    if (launch_permute(hid + bounds[c] * H, dst + bounds[c] * k, len(c), H, k, xy(c), L.rows_cap,
                       sm, dev_status) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaEventRecord(ctx->ev_perm[c & 1], sm) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  };
  auto experts = [&](int c) -> moe_status_t {
    // separate dispatch: wait for P(c); fused: wait until U(c-2) has read buffer c % 2
    if (!fused) {
      if (cudaStreamWaitEvent(sg, ctx->ev_perm[c & 1], 0) != cudaSuccess) return MOE_ERR_CUDA;
    } else if (c >= 2) {
      if (cudaStreamWaitEvent(sg, ctx->ev_unperm[c & 1], 0) != cudaSuccess) return MOE_ERR_CUDA;
    }
    const int64_t rows = len(c) * k;
    const int32_t* offs = reinterpret_cast<const int32_t*>(ws + L.offsets) + (size_t)c * (E + 1);
    moe_status_t s2 =
        fused ? gemm_call(nullptr, rows, W_gate_up, act(c), offs, nullptr, E, H, I, 2 * I, true,
                          dev_status, ctx->num_sms, sg, src + bounds[c] * k, hidden, T, c)
              : gemm_call(xy(c), rows, W_gate_up, act(c), offs, nullptr, E, H, I, 2 * I, true,
                          dev_status, ctx->num_sms, sg, nullptr, nullptr, 0, c);
    if (s2 != MOE_OK) return s2;
    s2 = gemm_call(act(c), rows, W_down, xy(c), offs, nullptr, E, I, H, H, false, dev_status,
                   ctx->num_sms, sg, nullptr, nullptr, 0, c);
    if (s2 != MOE_OK) return s2;
    if (cudaEventRecord(ctx->ev_gemm[c & 1], sg) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  };
  auto unpermute = [&](int c) -> moe_status_t {
    if (cudaStreamWaitEvent(sm, ctx->ev_gemm[c & 1], 0) != cudaSuccess) return MOE_ERR_CUDA;
    ProfScope ps(MOE_KERNEL_UNPERMUTE, sm, len(c) * k, 0, 1);
    if (launch_unpermute(xy(c), dst + bounds[c] * k, top_k_weights + bounds[c] * k, len(c), H, k,
                         outp + bounds[c] * H, L.rows_cap, sm, 0, dev_status) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (fused && cudaEventRecord(ctx->ev_unperm[c & 1], sm) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  };

  // 3) the pair pipeline
  if (n_live > 0 && !fused) {
    // M: P(0) P(1) U(0) P(2) U(1) ...; G: E(0) E(1) E(2) ...
    if ((st = permute(0)) != MOE_OK || (st = experts(0)) != MOE_OK) return st;
    for (int c = 0; c < n_live; ++c) {
      if (c + 1 < n_live) {
        if ((st = permute(c + 1)) != MOE_OK || (st = experts(c + 1)) != MOE_OK) return st;
      }
      if ((st = unpermute(c)) != MOE_OK) return st;
    }
  } else if (n_live > 0 && pair_gemms) {
    // Pairs (c0, c1) = (2m, 2m+1).  M: GU(m) D(m) GU(m+1) D(m+1) ... U(last), where GU / D
    // are the gate/up and down GEMMs of the pair in one tile sweep over its rows, laid out
    // per expert across both chunks (each expert's weight tiles are fetched once for the
    // pair, and a row tile may hold rows of both chunks), and U the combine of both chunks
    // of a pair in one launch; G: U(m) after D(m), beside GU(m+1), for every pair but the
    // last.  D(m+1) waits until U(m) has read the pair's Y rows.  The GEMMs and the last
    // combine follow the metadata on the caller's stream, so that no launch on the critical
    // path waits for another stream.  The pair's rows fill both halves of the X|Y and Act
    // double buffers; dst holds pair-local rows.
    const std::vector<int64_t> pb = dims_bounds(dm);
    void* y_pair = ws + L.xy[0];
    void* act_pair = ws + L.act[0];
    const int64_t pair_cap = L.rows_cap * L.nbuf;
    for (int m = 0; 2 * m < n_live; ++m) {
      const int c0 = 2 * m, c1 = 2 * m + 1 < n_live ? 2 * m + 1 : 2 * m;
      NvtxRange pr("moe_forward pair: chunks %d-%d", c0, c1);
      const int64_t rows = (pb[m + 1] - pb[m]) * k;
      const int32_t* offs = reinterpret_cast<const int32_t*>(ws + L.offsets) + (size_t)m * (E + 1);
      moe_status_t s2 = gemm_call(nullptr, rows, W_gate_up, act_pair, offs, nullptr, E, H, I,
                                  2 * I, true, dev_status, ctx->num_sms, sm, src + pb[m] * k,
                                  hidden, T, m);
      if (s2 != MOE_OK) return s2;
      if (m > 0 && cudaStreamWaitEvent(sm, ctx->ev_unperm[0], 0) != cudaSuccess)
        return MOE_ERR_CUDA;
      s2 = gemm_call(act_pair, rows, W_down, y_pair, offs, nullptr, E, I, H, H, false, dev_status,
                     ctx->num_sms, sm, nullptr, nullptr, 0, m);
      if (s2 != MOE_OK) return s2;
      // a pair's combine runs on the side stream beside the next pair's gate/up GEMM (fewer
      // CTAs, all resident next to it) unless this is the last pair
      // (one launch for both chunks: their tokens are adjacent and dst holds pair-local rows)
      const bool beside_gemm = 2 * (m + 1) < n_live;
      cudaStream_t su = beside_gemm ? sg : sm;
      if (beside_gemm && (cudaEventRecord(ctx->ev_gemm[0], sm) != cudaSuccess ||
                          cudaStreamWaitEvent(sg, ctx->ev_gemm[0], 0) != cudaSuccess))
        return MOE_ERR_CUDA;
      {
        const int64_t t0 = bounds[c0], tn = bounds[c1 + 1] - bounds[c0];
        ProfScope ps(MOE_KERNEL_UNPERMUTE, su, tn * k, 0, 1);
        if (launch_unpermute(y_pair, dst + t0 * k, top_k_weights + t0 * k, tn, H, k,
                             outp + t0 * H, pair_cap, su,
                             beside_gemm ? MOE_UNPERM_BESIDE_GEMM_CTAS_PER_SM : 0,
                             dev_status) != cudaSuccess)
          return MOE_ERR_CUDA;
      }
      if (beside_gemm && cudaEventRecord(ctx->ev_unperm[0], sg) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
  } else if (n_live > 0) {
    // G: E(0) E(1) E(2) ... (E(c+2) after U(c) freed buffer c % 2); M: U(0) U(1) ...
    if ((st = experts(0)) != MOE_OK) return st;
    if (n_live > 1 && (st = experts(1)) != MOE_OK) return st;
    for (int c = 0; c < n_live; ++c) {
      if ((st = unpermute(c)) != MOE_OK) return st;
      if (c + 2 < n_live && (st = experts(c + 2)) != MOE_OK) return st;
    }
  }
  if (cudaEventRecord(ctx->ev_join, sg) != cudaSuccess ||
      cudaStreamWaitEvent(sm, ctx->ev_join, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  // the metadata's host copy (enqueued right after it, long done by now on the device)
  st = fetch_packed_wait(ctx);
  if (g_prof.on) prof_fix_active(ctx->host_stage + kStatusWords, E);
  return st;
}

size_t moe_workspace_bytes_host(const moe_shape_t* s) {
  if (check_shape(s) != MOE_OK) return 0;
  const Dims d = make_dims(s->T, s->k, s->E, s->ep_groups, s->num_chunks, s->chunk_size);
  const Layout L = make_layout(d, s->H, s->I, true, true, true);
  return make_host_staging(d, s->H, L.total).total;
}

moe_status_t moe_forward_host_impl(const moe_shape_t* shape, const void* hidden_host,
                                   const int32_t* top_k_index_host,
                                   const float* top_k_weights_host, const void* W_gate_up,
                                   const void* W_down, void* out_host, void* workspace,
                                   size_t ws_bytes, void* stream);

moe_status_t moe_forward_host(const moe_shape_t* shape, const void* hidden_host,
                              const int32_t* top_k_index_host, const float* top_k_weights_host,
                              const void* W_gate_up, const void* W_down, void* out_host,
                              void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange range("moe_forward_host");
  ProfCall prof_call;
  return moe_forward_host_impl(shape, hidden_host, top_k_index_host, top_k_weights_host,
                               W_gate_up, W_down, out_host, workspace, ws_bytes, stream);
}

moe_status_t moe_forward_host_impl(const moe_shape_t* shape, const void* hidden_host,
                              const int32_t* top_k_index_host, const float* top_k_weights_host,
                              const void* W_gate_up, const void* W_down, void* out_host,
                              void* workspace, size_t ws_bytes, void* stream) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  const int64_t T = shape->T;
  const int32_t H = shape->H, I = shape->I, E = shape->E, k = shape->k;
  if (T == 0) return MOE_OK;
  if (!hidden_host || !top_k_index_host || !top_k_weights_host || !W_gate_up || !W_down ||
      !out_host || !workspace)
    return MOE_ERR_ARG;
  if (!aligned(W_gate_up, 16) || !aligned(W_down, 16) || !aligned(workspace, kAlign) ||
      !aligned(top_k_index_host, 4) || !aligned(top_k_weights_host, 4) ||
      !aligned(hidden_host, 2) || !aligned(out_host, 2))
    return MOE_ERR_ALIGN;
  const Dims d = make_dims(T, k, E, shape->ep_groups, shape->num_chunks, shape->chunk_size);
  const Layout L = make_layout(d, H, I, true, true, true);
  const HostStaging hs = make_host_staging(d, H, L.total);
  if (ws_bytes < hs.total) return MOE_ERR_WORKSPACE;
  DeviceCtx* ctx = nullptr;
  if ((st = get_ctx(&ctx)) != MOE_OK) return st;
  cudaStream_t sm = static_cast<cudaStream_t>(stream);
  cudaStream_t sg = ctx->side, ci = ctx->copy_in, co = ctx->copy_out;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* dst = reinterpret_cast<int32_t*>(ws + L.dst);
  int32_t* src = reinterpret_cast<int32_t*>(ws + L.src);
  uint32_t* dev_status = reinterpret_cast<uint32_t*>(ws + L.packed);
  int32_t* idx_dev = reinterpret_cast<int32_t*>(ws + hs.idx);
  float* w_dev = reinterpret_cast<float*>(ws + hs.w);
  const size_t row_bytes = sizeof(uint16_t) * (size_t)H;
  const uint8_t* hid_h = static_cast<const uint8_t*>(hidden_host);
  uint8_t* out_h = static_cast<uint8_t*>(out_host);

  // routing arrays first: the metadata of every chunk needs all of them
  if (cudaMemcpyAsync(idx_dev, top_k_index_host, sizeof(int32_t) * (size_t)(T * k),
                      cudaMemcpyHostToDevice, sm) != cudaSuccess ||
      cudaMemcpyAsync(w_dev, top_k_weights_host, sizeof(float) * (size_t)(T * k),
                      cudaMemcpyHostToDevice, sm) != cudaSuccess)
    return MOE_ERR_CUDA;
  std::vector<int64_t> bounds = dims_bounds(d);
  int n_live = 0;
  while (n_live < d.n && bounds[n_live + 1] > bounds[n_live]) ++n_live;
  auto len = [&](int c) { return bounds[c + 1] - bounds[c]; };
  // copy-in of chunk c into input buffer c % 2 (after P(c-2) has read it)
  auto copy_in = [&](int c) -> moe_status_t {
    if (c >= 2 && cudaStreamWaitEvent(ci, ctx->ev_in_free[c & 1], 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(ws + hs.in[c & 1], hid_h + bounds[c] * row_bytes, len(c) * row_bytes,
                        cudaMemcpyHostToDevice, ci) != cudaSuccess ||
        cudaEventRecord(ctx->ev_in[c & 1], ci) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  };
  // the first two chunks' rows can travel while the metadata runs
  if (cudaEventRecord(ctx->ev_start, sm) != cudaSuccess ||
      cudaStreamWaitEvent(ci, ctx->ev_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(co, ctx->ev_start, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int c = 0; c < n_live && c < 2; ++c)
    if ((st = copy_in(c)) != MOE_OK) return st;

  // Fused dispatch (gate/up GEMM gathering its rows from the chunk's staged input) where one
  // chunk's permuted copy would be a sizeable share of the GEMM traffic, as moe_forward
  // decides for one chunk; the gather map then indexes the chunk's own rows.
  const bool fused = 4 * d.t_chunk * d.k >= (int64_t)d.E * shape->I;
  if ((st = run_metadata(d, idx_dev, ws, L, dst, src, sm, fused)) != MOE_OK) return st;
  if ((st = fetch_packed(ctx, ws, L, sm)) != MOE_OK) return st;
  std::vector<int32_t> counts(ctx->host_stage + kStatusWords,
                              ctx->host_stage + kStatusWords + (size_t)d.n * d.E);

  auto xy = [&](int c) { return ws + L.xy[c % L.nbuf]; };
  auto act = [&](int c) { return ws + L.act[c % L.nbuf]; };
  auto permute = [&](int c) -> moe_status_t {
    if (cudaStreamWaitEvent(sm, ctx->ev_in[c & 1], 0) != cudaSuccess) return MOE_ERR_CUDA;
    {
      ProfScope ps(MOE_KERNEL_PERMUTE, sm, len(c) * k, 0, 1);
      if (launch_permute(ws + hs.in[c & 1], dst + bounds[c] * k, len(c), H, k, xy(c), L.rows_cap,
                         sm) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    if (cudaEventRecord(ctx->ev_perm[c & 1], sm) != cudaSuccess ||
        cudaEventRecord(ctx->ev_in_free[c & 1], sm) != cudaSuccess)
      return MOE_ERR_CUDA;
    return c + 2 < n_live ? copy_in(c + 2) : MOE_OK;
  };
  auto experts = [&](int c) -> moe_status_t {
    if (cudaStreamWaitEvent(sg, ctx->ev_perm[c & 1], 0) != cudaSuccess) return MOE_ERR_CUDA;
    const int64_t rows = len(c) * k;
    const int32_t* cnt = counts.data() + (size_t)c * E;
    const int32_t* offs = reinterpret_cast<const int32_t*>(ws + L.offsets) + (size_t)c * (E + 1);
    moe_status_t s2 = gemm_call(xy(c), rows, W_gate_up, act(c), offs, cnt, E, H, I, 2 * I, true,
                                dev_status, ctx->num_sms, sg);
    if (s2 != MOE_OK) return s2;
    s2 = gemm_call(act(c), rows, W_down, xy(c), offs, cnt, E, I, H, H, false, dev_status,
                   ctx->num_sms, sg);
    if (s2 != MOE_OK) return s2;
    return cudaEventRecord(ctx->ev_gemm[c & 1], sg) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  };
  // fused: chunk c's GEMMs gather from input buffer c % 2, which they free after the
  // gate/up GEMM (the copy-in of chunk c+2 waits for that); buffer c % 2 of the expert rows
  // is free once U(c-2) has read it
  auto experts_fused = [&](int c) -> moe_status_t {
    if (cudaStreamWaitEvent(sg, ctx->ev_in[c & 1], 0) != cudaSuccess ||
        (c >= 2 && cudaStreamWaitEvent(sg, ctx->ev_unperm[c & 1], 0) != cudaSuccess))
      return MOE_ERR_CUDA;
    const int64_t rows = len(c) * k;
    const int32_t* cnt = counts.data() + (size_t)c * E;
    const int32_t* offs = reinterpret_cast<const int32_t*>(ws + L.offsets) + (size_t)c * (E + 1);
    moe_status_t s2 = gemm_call(nullptr, rows, W_gate_up, act(c), offs, cnt, E, H, I, 2 * I, true,
                                dev_status, ctx->num_sms, sg, src + bounds[c] * k,
                                ws + hs.in[c & 1], len(c));
    if (s2 != MOE_OK) return s2;
    if (cudaEventRecord(ctx->ev_in_free[c & 1], sg) != cudaSuccess) return MOE_ERR_CUDA;
    s2 = gemm_call(act(c), rows, W_down, xy(c), offs, cnt, E, I, H, H, false, dev_status,
                   ctx->num_sms, sg);
    if (s2 != MOE_OK) return s2;
    if (cudaEventRecord(ctx->ev_gemm[c & 1], sg) != cudaSuccess) return MOE_ERR_CUDA;
    return c + 2 < n_live ? copy_in(c + 2) : MOE_OK;
  };
  auto unpermute = [&](int c) -> moe_status_t {
    if (cudaStreamWaitEvent(sm, ctx->ev_gemm[c & 1], 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (c >= 2 && cudaStreamWaitEvent(sm, ctx->ev_out_free[c & 1], 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    {
      ProfScope ps(MOE_KERNEL_UNPERMUTE, sm, len(c) * k, 0, 1);
      if (launch_unpermute(xy(c), dst + bounds[c] * k, w_dev + bounds[c] * k, len(c), H, k,
                           ws + hs.out[c & 1], L.rows_cap, sm) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    if (fused && cudaEventRecord(ctx->ev_unperm[c & 1], sm) != cudaSuccess) return MOE_ERR_CUDA;
    // copy-out of chunk c beside the next chunk's GEMMs
    if (cudaEventRecord(ctx->ev_out[c & 1], sm) != cudaSuccess ||
        cudaStreamWaitEvent(co, ctx->ev_out[c & 1], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_h + bounds[c] * row_bytes, ws + hs.out[c & 1], len(c) * row_bytes,
                        cudaMemcpyDeviceToHost, co) != cudaSuccess ||
        cudaEventRecord(ctx->ev_out_free[c & 1], co) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  };

  if (cudaEventRecord(ctx->ev_start, sm) != cudaSuccess ||
      cudaStreamWaitEvent(sg, ctx->ev_start, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (n_live > 0 && fused) {
    // G: E(0) E(1) E(2) ... (E(c+2) after U(c) freed buffer c % 2); M: U(0) U(1) ...
    if ((st = experts_fused(0)) != MOE_OK) return st;
    if (n_live > 1 && (st = experts_fused(1)) != MOE_OK) return st;
    for (int c = 0; c < n_live; ++c) {
      if ((st = unpermute(c)) != MOE_OK) return st;
      if (c + 2 < n_live && (st = experts_fused(c + 2)) != MOE_OK) return st;
    }
  } else if (n_live > 0) {
    if ((st = permute(0)) != MOE_OK || (st = experts(0)) != MOE_OK) return st;
    for (int c = 0; c < n_live; ++c) {
      if (c + 1 < n_live) {
        if ((st = permute(c + 1)) != MOE_OK || (st = experts(c + 1)) != MOE_OK) return st;
      }
      if ((st = unpermute(c)) != MOE_OK) return st;
    }
  }
  // join every stream into `stream` and wait for out_host
  if (cudaEventRecord(ctx->ev_join, sg) != cudaSuccess ||
      cudaStreamWaitEvent(sm, ctx->ev_join, 0) != cudaSuccess ||
      cudaEventRecord(ctx->ev_copy_join, co) != cudaSuccess ||
      cudaStreamWaitEvent(sm, ctx->ev_copy_join, 0) != cudaSuccess ||
      cudaStreamSynchronize(sm) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// ---- backward -------------------------------------------------------------------------

namespace {

struct BwdLayout {
  Dims unit;    // the pairs of chunks (2m, 2m+1), each a unit of the pipeline
  Layout meta;  // metadata regions (status/counts/splits, offsets, histograms, dst, src)
  size_t offp, first, dstp, total;
  int nx;  // X buffers: one per pair in flight (up to 2)
  size_t xp[2], wrow[2];  // X rows and their routing weights, per pair in flight
  size_t gu, act, dx, dy;  // gu later holds [dg du] in place
  size_t dwp;              // partial d_w of each row
  int32_t dw_slots;
  int64_t rows_cap;
};

// The backward runs per pair of chunks: the metadata is taken per pair, so each expert's
// rows are contiguous over both chunks and padded once per pair to a multiple of 64; every
// pair's rows fit in rows_cap rows.  The pipeline keeps pair m's permuted rows and their
// routing weights in buffer set m % 2 (the next pair is permuted while pair m computes; X is
// read until the pair's weight-gradient GEMM) and its other rows in one buffer set.  The SwiGLU backward
// overwrites the saved [g u] rows with [dg du] (each epilogue thread has read a block before
// any lane stores it), so one buffer holds both.
BwdLayout make_bwd_layout(const Dims& d, int32_t H, int32_t I) {
  BwdLayout B{};
  B.unit = pair_dims(d);
  const Dims& u = B.unit;
  B.meta = make_layout(u, 8, 8, false, true, true);
  size_t o = B.meta.total;
  B.rows_cap = u.t_chunk * u.k + (int64_t)u.E * (bwd_pad_rows() - 1);
  B.offp = o;
  o += al(sizeof(int32_t) * (size_t)u.n * (u.E + 1));
  B.first = o;
  o += al(sizeof(int32_t) * (size_t)u.E);
  B.dstp = o;
  o += al(sizeof(int32_t) * (size_t)(u.T * u.k));
  const size_t R = (size_t)B.rows_cap;
  B.nx = u.n >= 2 ? 2 : 1;
  for (int b = 0; b < B.nx; ++b) {
    B.xp[b] = o;
    o += al(2 * R * H);
    B.wrow[b] = o;
    o += al(sizeof(float) * R);
  }
  B.gu = o;
  o += al(2 * R * 2 * I);
  B.act = o;
  o += al(2 * R * I);
  B.dx = o;
  o += al(2 * R * H);
  B.dy = o;
  o += al(2 * R * H);
  B.dw_slots = bwd_dw_slots(I);
  B.dwp = o;
  o += al(sizeof(float) * R * B.dw_slots);
  B.total = o;
  return B;
}

moe_status_t check_bwd_shape(const moe_shape_t* s) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (s->H % 64 != 0 || s->I % 32 != 0) return MOE_ERR_ARG;
  return MOE_OK;
}

}  // namespace

size_t moe_backward_workspace_bytes(const moe_shape_t* s) {
  if (check_bwd_shape(s) != MOE_OK) return 0;
  const Dims d = make_dims(s->T, s->k, s->E, s->ep_groups, s->num_chunks, s->chunk_size);
  return make_bwd_layout(d, s->H, s->I).total;
}

moe_status_t moe_backward(const moe_shape_t* shape, const void* hidden,
                          const int32_t* top_k_index, const float* top_k_weights,
                          const void* W_gate_up, const void* W_down, const void* d_out,
                          void* d_hidden, float* d_weights, float* dW_gate_up, float* dW_down,
                          void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange range("moe_backward");
  ProfCall prof_call;
  moe_status_t st = check_bwd_shape(shape);
  if (st != MOE_OK) return st;
  const int64_t T = shape->T;
  const int32_t H = shape->H, I = shape->I, E = shape->E, k = shape->k;
  if (!W_gate_up || !W_down || !dW_gate_up || !dW_down) return MOE_ERR_ARG;
  if (T > 0 && (!hidden || !top_k_index || !top_k_weights || !d_out || !d_hidden ||
                !d_weights || !workspace))
    return MOE_ERR_ARG;
  if (!aligned(hidden, 16) || !aligned(d_out, 16) || !aligned(d_hidden, 16) ||
      !aligned(W_gate_up, 16) || !aligned(W_down, 16) || !aligned(dW_gate_up, 16) ||
      !aligned(dW_down, 16) || !aligned(top_k_index, 4) || !aligned(top_k_weights, 4) ||
      !aligned(d_weights, 4) || !aligned(workspace, kAlign))
    return MOE_ERR_ALIGN;
  const Dims d = make_dims(T, k, E, shape->ep_groups, shape->num_chunks, shape->chunk_size);
  const BwdLayout B = make_bwd_layout(d, H, I);
  if (T > 0 && ws_bytes < B.total) return MOE_ERR_WORKSPACE;
  DeviceCtx* ctx = nullptr;
  if ((st = get_ctx(&ctx)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t gu_per_e = (size_t)2 * I * H, dn_per_e = (size_t)H * I;  // fp32 elements
  auto zero_experts = [&](int32_t e0, int32_t e1) {
    return cudaMemsetAsync(dW_gate_up + e0 * gu_per_e, 0, sizeof(float) * (e1 - e0) * gu_per_e,
                           s) == cudaSuccess &&
           cudaMemsetAsync(dW_down + e0 * dn_per_e, 0, sizeof(float) * (e1 - e0) * dn_per_e, s) ==
               cudaSuccess;
  };
  if (T == 0) return zero_experts(0, E) ? MOE_OK : MOE_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* dst = reinterpret_cast<int32_t*>(ws + B.meta.dst);
  int32_t* src = reinterpret_cast<int32_t*>(ws + B.meta.src);
  uint32_t* dev_status = reinterpret_cast<uint32_t*>(ws + B.meta.packed);
  const Dims& u = B.unit;  // unit m = the pair of chunks (2m, 2m+1)
  if ((st = run_metadata(u, top_k_index, ws, B.meta, dst, src, s)) != MOE_OK) return st;
  if ((st = fetch_packed(ctx, ws, B.meta, s)) != MOE_OK) return st;
  std::vector<int32_t> counts(ctx->host_stage + kStatusWords,
                              ctx->host_stage + kStatusWords + (size_t)u.n * E);
  const int32_t* counts_dev = reinterpret_cast<const int32_t*>(ws + B.meta.packed) + kStatusWords;
  int32_t* offp = reinterpret_cast<int32_t*>(ws + B.offp);
  int32_t* first = reinterpret_cast<int32_t*>(ws + B.first);
  int32_t* dstp = reinterpret_cast<int32_t*>(ws + B.dstp);
  if (launch_pad_offsets(counts_dev, E, u.n, offp, first, s) != cudaSuccess) return MOE_ERR_CUDA;
  // The weight-gradient GEMM of an expert's first pair with rows stores its tiles and later
  // pairs add to them, so only experts that no chunk routes to are zeroed here (runs of
  // consecutive such experts take one memset per gradient).
  std::vector<char> routed((size_t)E, 0);
  for (int m = 0; m < u.n; ++m)
    for (int32_t e = 0; e < E; ++e) routed[e] |= counts[(size_t)m * E + e] > 0;
  for (int32_t e0 = 0; e0 < E;) {
    if (routed[e0]) {
      ++e0;
      continue;
    }
    int32_t e1 = e0 + 1;
    while (e1 < E && !routed[e1]) ++e1;
    if (!zero_experts(e0, e1)) return MOE_ERR_CUDA;
    e0 = e1;
  }
  const std::vector<int64_t> bounds = dims_bounds(u);
  int n_live = 0;  // pairs with tokens; only trailing ones can be empty
  while (n_live < u.n && bounds[n_live + 1] > bounds[n_live]) ++n_live;
  const int pad = bwd_pad_rows();
  const uint16_t* hid = static_cast<const uint16_t*>(hidden);
  const uint16_t* dout = static_cast<const uint16_t*>(d_out);
  uint16_t* dx_out = static_cast<uint16_t*>(d_hidden);
  cudaStream_t sg = ctx->side;
  // padded rows per expert and their total, per pair
  std::vector<int32_t> rows_pad((size_t)u.n * E);
  std::vector<int64_t> R((size_t)u.n, 0);
  for (int m = 0; m < u.n; ++m)
    for (int32_t e = 0; e < E; ++e) {
      const int32_t v = (counts[(size_t)m * E + e] + pad - 1) / pad * pad;
      rows_pad[(size_t)m * E + e] = v;
      R[m] += v;
    }
  auto x_of = [&](int m) { return ws + B.xp[m % B.nx]; };
  auto wrow_of = [&](int m) { return reinterpret_cast<float*>(ws + B.wrow[m % B.nx]); };
  uint8_t* const gu = ws + B.gu;    // [g u], later [dg du]
  uint8_t* const act = ws + B.act;  // w h
  uint8_t* const dxr = ws + B.dx;   // dX
  uint8_t* const dy = ws + B.dy;    // dY: the dout row of each copy
  float* const dwp = reinterpret_cast<float*>(ws + B.dwp);
  auto off_m = [&](int m) {
    return reinterpret_cast<const int32_t*>(ws + B.meta.offsets) + (size_t)m * (E + 1);
  };
  auto offp_m = [&](int m) -> const int32_t* { return offp + (size_t)m * (E + 1); };
  auto rows_pad_m = [&](int m) { return rows_pad.data() + (size_t)m * E; };
  auto dstp_m = [&](int m) { return dstp + bounds[m] * k; };
  auto len = [&](int m) { return bounds[m + 1] - bounds[m]; };
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };

  // P(m), stream M: padded permute of the pair's rows into X buffer m % 2 and their routing
  // weights into the weight buffer m % 2 (zero pad rows), once W(m-2) is done with them
  auto P = [&](int m) -> moe_status_t {
    if (m >= 2 && !ok(cudaStreamWaitEvent(s, ctx->ev_bw[m % 2], 0))) return MOE_ERR_CUDA;
    ProfScope ps(MOE_KERNEL_BWD_ROWS, s, len(m) * k, 0, 3);
    if (!ok(launch_zero_pad_rows(off_m(m), offp_m(m), E, H, x_of(m), wrow_of(m), B.rows_cap,
                                 s)) ||
        !ok(launch_pad_rows(top_k_index + bounds[m] * k, dst + bounds[m] * k, off_m(m),
                            offp_m(m), top_k_weights + bounds[m] * k, len(m) * k, dstp_m(m),
                            wrow_of(m), B.rows_cap, s)) ||
        !ok(launch_permute(hid + bounds[m] * H, dstp_m(m), len(m), H, k, x_of(m), B.rows_cap,
                           s)) ||
        !ok(cudaEventRecord(ctx->ev_bp[m % 2], s)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  };
  BwdGemmArgs g0{};
  g0.E = E;
  g0.I = I;
  g0.status = dev_status;
  g0.first = first;
  // A GEMM over the pair's padded rows: one tile sweep per pair, so each weight tile is
  // fetched once for both chunks, and a row tile may hold rows of both.
  auto rowwise = [&](int m, int mode) {
    BwdGemmArgs g = g0;
    g.mode = mode;
    g.offsets = offp_m(m);
    g.rows_pad_host = rows_pad_m(m);
    g.chunk = m;
    return g;
  };
  auto launch_unit = [&](int kind, const BwdGemmArgs& a, int m) {
    ProfScope ps(kind, sg, R[m], active_experts(rows_pad_m(m), E), 1);
    return launch_bwd_gemm(a, ctx->num_sms, sg);
  };
  // F(m), stream G: recompute [g u] and w h on the padded rows, once P(m) is done
  auto F = [&](int m) -> moe_status_t {
    if (!ok(cudaStreamWaitEvent(sg, ctx->ev_bp[m % 2], 0))) return MOE_ERR_CUDA;
    BwdGemmArgs g = rowwise(m, kBwdRawGU);
    g.A = x_of(m), g.A_rows = R[m], g.A_cols = H;
    g.B = W_gate_up, g.B_rows = (int64_t)E * 2 * I, g.B_cols = H;
    g.N = 2 * I, g.K = H, g.b_rows = 2 * I, g.out0 = gu, g.out1 = act, g.wrow = wrow_of(m);
    return ok(launch_unit(MOE_KERNEL_BWD_GATEUP, g, m)) ? MOE_OK : MOE_ERR_CUDA;
  };
  // DYS(m), stream M: the dout row of each copy into the pair's padded dY rows (zero pad
  // rows); it needs nothing from the recompute, only the previous pair's weight gradients to
  // be done with the dY rows
  auto DYS = [&](int m) -> moe_status_t {
    ProfScope ps(MOE_KERNEL_BWD_ROWS, s, len(m) * k, 0, 2);
    if (!ok(launch_zero_pad_rows(off_m(m), offp_m(m), E, H, dy, nullptr, B.rows_cap, s)) ||
        !ok(launch_permute(dout + bounds[m] * H, dstp_m(m), len(m), H, k, dy, B.rows_cap, s)) ||
        !ok(cudaEventRecord(ctx->ev_bdy[0], s)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  };
  // DW(m), stream M: d_weights = the sum of each copy's partials, once the SwiGLU-backward
  // GEMM of the pair has written them
  auto DW = [&](int m) -> moe_status_t {
    if (!ok(cudaStreamWaitEvent(s, ctx->ev_bdy[1], 0))) return MOE_ERR_CUDA;
    ProfScope ps(MOE_KERNEL_BWD_ROWS, s, len(m) * k, 0, 1);
    if (!ok(launch_dw_sum(dwp, dstp_m(m), len(m) * k, B.dw_slots, d_weights + bounds[m] * k,
                          B.rows_cap, s)) ||
        !ok(cudaEventRecord(ctx->ev_bf[0], s)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  };
  // Bd(m), stream G: the SwiGLU backward (dg, du and the partials of d_w), once the pair's dY
  // rows are in and DW(m-1) has read the previous partials; then dX, once S(m-1) has read
  // the previous pair's dX rows
  auto Bd = [&](int m) -> moe_status_t {
    if (!ok(cudaStreamWaitEvent(sg, ctx->ev_bdy[0], 0))) return MOE_ERR_CUDA;  // dY rows
    if (m >= 1 && !ok(cudaStreamWaitEvent(sg, ctx->ev_bf[0], 0))) return MOE_ERR_CUDA;
    BwdGemmArgs g = rowwise(m, kBwdDSwiGLU);
    g.A = dy, g.A_rows = R[m], g.A_cols = H;
    g.B = W_down, g.B_rows = (int64_t)E * H, g.B_cols = I;
    g.N = I, g.K = H, g.b_rows = H, g.out0 = gu, g.aux = gu;  // in place
    g.wrow = wrow_of(m), g.dwp = dwp;
    if (!ok(launch_unit(MOE_KERNEL_BWD_DSWIGLU, g, m)) ||
        !ok(cudaEventRecord(ctx->ev_bdy[1], sg)))
      return MOE_ERR_CUDA;
    if (m >= 1 && !ok(cudaStreamWaitEvent(sg, ctx->ev_bsum[0], 0))) return MOE_ERR_CUDA;
    g = rowwise(m, kBwdDPlain);
    g.A = gu, g.A_rows = R[m], g.A_cols = 2 * I;
    g.B = W_gate_up, g.B_rows = (int64_t)E * 2 * I, g.B_cols = H;
    g.N = H, g.K = 2 * I, g.b_rows = 2 * I, g.out0 = dxr;
    if (!ok(launch_unit(MOE_KERNEL_BWD_DX, g, m)) || !ok(cudaEventRecord(ctx->ev_bdx[0], sg)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  };
  // W(m), stream G: both weight gradients, K over the pair's padded rows:
  //   dW_down[e] (+)= dY^T (w h) ;  dW_gate_up[e] (+)= [dg du]^T X
  // An expert's first pair with rows stores; later pairs add.
  auto W = [&](int m) -> moe_status_t {
    BwdGemmArgs g = rowwise(m, kBwdWGrad);
    g.A = dy, g.A_rows = R[m], g.A_cols = H;
    g.B = act, g.B_rows = R[m], g.B_cols = I;
    g.M = H, g.N = I, g.acc = dW_down, g.out0 = nullptr;
    if (!ok(launch_unit(MOE_KERNEL_BWD_WGRAD, g, m))) return MOE_ERR_CUDA;
    g.A = gu, g.A_rows = R[m], g.A_cols = 2 * I;  // [dg du]
    g.B = x_of(m), g.B_rows = R[m], g.B_cols = H;
    g.M = 2 * I, g.N = H, g.acc = dW_gate_up;
    if (!ok(launch_unit(MOE_KERNEL_BWD_WGRAD, g, m)) ||
        !ok(cudaEventRecord(ctx->ev_bw[m % 2], sg)) || !ok(cudaEventRecord(ctx->ev_bf[1], sg)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  };
  // S(m), stream M: d_hidden rows = sum over the k copies of dX
  auto S = [&](int m) -> moe_status_t {
    if (!ok(cudaStreamWaitEvent(s, ctx->ev_bdx[0], 0))) return MOE_ERR_CUDA;
    ProfScope ps(MOE_KERNEL_BWD_ROWS, s, len(m) * k, 0, 1);
    if (!ok(launch_sum_rows(dxr, dstp_m(m), len(m), H, k, dx_out + bounds[m] * H, B.rows_cap,
                            s)) ||
        !ok(cudaEventRecord(ctx->ev_bsum[0], s)))
      return MOE_ERR_CUDA;
    return MOE_OK;
  };

  // The mirrored pair pipeline, one unit per pair of chunks:
  //   G: F(0) DSwiGLU(0) DX(0) W(0) F(1) DSwiGLU(1) ...
  //   M: P(0) DYS(0) | P(1) DW(0) S(0) DYS(1) | P(2) DW(1) S(1) ...
  // dY needs nothing from the recompute, so it is scattered while F runs; the next pair is
  // permuted beside the SwiGLU-backward GEMM, d_weights is summed beside the dX GEMM, and
  // the next pair's dY is scattered once W(m) is done with the dY rows.  Host enqueue order
  // keeps each event wait on the record it is meant for.
  if (!ok(cudaEventRecord(ctx->ev_start, s)) || !ok(cudaStreamWaitEvent(sg, ctx->ev_start, 0)))
    return MOE_ERR_CUDA;
  if (n_live > 0) {
    if ((st = P(0)) != MOE_OK || (st = F(0)) != MOE_OK || (st = DYS(0)) != MOE_OK) return st;
    for (int m = 0; m < n_live; ++m) {
      NvtxRange pr("moe_backward pair %d", m, 0);
      if (m + 1 < n_live && (st = P(m + 1)) != MOE_OK) return st;
      if ((st = Bd(m)) != MOE_OK || (st = DW(m)) != MOE_OK || (st = S(m)) != MOE_OK ||
          (st = W(m)) != MOE_OK)
        return st;
      if (m + 1 < n_live) {
        if ((st = F(m + 1)) != MOE_OK) return st;
        if (!ok(cudaStreamWaitEvent(s, ctx->ev_bf[1], 0))) return MOE_ERR_CUDA;  // W(m) done
        if ((st = DYS(m + 1)) != MOE_OK) return st;
      }
    }
  }
  if (!ok(cudaEventRecord(ctx->ev_join, sg)) || !ok(cudaStreamWaitEvent(s, ctx->ev_join, 0)))
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int32_t moe_checks_enabled(void) { return MOE_CHECKS ? 1 : 0; }

moe_status_t moe_checks_read(uint32_t* flags) {
  if (!flags) return MOE_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  *flags = checks_take_permute() | checks_take_gemm() | checks_take_backward() |
           checks_take_ep();
  return MOE_OK;
}

moe_status_t moe_check_device_status(const void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < sizeof(uint32_t)) return MOE_ERR_ARG;
  uint32_t st = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, workspace, sizeof st, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (st & MOE_DEV_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (st & MOE_DEV_BAD_INDEX) return MOE_ERR_INDEX;
  return MOE_OK;
}

moe_status_t moe_permute(const void* hidden, const int32_t* dst_rows, int64_t Tc, int32_t H,
                         int32_t k, void* X, void* stream) {
  if (Tc < 0 || H <= 0 || H % 8 || k <= 0 || k > MOE_MAX_TOPK) return MOE_ERR_ARG;
  if (Tc == 0) return MOE_OK;
  if (!hidden || !dst_rows || !X) return MOE_ERR_ARG;
  if (!aligned(hidden, 16) || !aligned(X, 16) || !aligned(dst_rows, 4)) return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ProfScope ps(MOE_KERNEL_PERMUTE, s, Tc * k, 0, 1);
  return cuda_status(launch_permute(hidden, dst_rows, Tc, H, k, X, Tc * k, s));
}

moe_status_t moe_unpermute(const void* Y, const int32_t* dst_rows, const float* top_k_weights,
                           int64_t Tc, int32_t H, int32_t k, void* out, void* stream) {
  if (Tc < 0 || H <= 0 || H % 8 || k <= 0 || k > MOE_MAX_TOPK) return MOE_ERR_ARG;
  if (Tc == 0) return MOE_OK;
  if (!Y || !dst_rows || !top_k_weights || !out) return MOE_ERR_ARG;
  if (!aligned(Y, 16) || !aligned(out, 16) || !aligned(dst_rows, 4) || !aligned(top_k_weights, 4))
    return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ProfScope ps(MOE_KERNEL_UNPERMUTE, s, Tc * k, 0, 1);
  return cuda_status(launch_unpermute(Y, dst_rows, top_k_weights, Tc, H, k, out, Tc * k, s));
}

static moe_status_t grouped_common(const void* A, int64_t rows, int32_t H, int32_t I, int32_t E,
                                   const int32_t* offsets, const int32_t* counts_host,
                                   const void* W, void* out, uint32_t* status, void* stream,
                                   bool swiglu) {
  if (rows < 0 || H <= 0 || I <= 0 || H % 8 || I % 8 || E <= 0) return MOE_ERR_ARG;
  if (E > MOE_MAX_EXPERTS || rows >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!A || !offsets || !counts_host || !W || !out || !status) return MOE_ERR_ARG;
  if (!aligned(A, 16) || !aligned(W, 16) || !aligned(out, 16) || !aligned(offsets, 4) ||
      !aligned(status, 4))
    return MOE_ERR_ALIGN;
  int64_t sum = 0;
  for (int32_t e = 0; e < E; ++e) {
    if (counts_host[e] < 0) return MOE_ERR_ARG;
    sum += counts_host[e];
  }
  if (sum != rows) return MOE_ERR_ARG;
  DeviceCtx* ctx = nullptr;
  moe_status_t st = get_ctx(&ctx);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (swiglu)
    return gemm_call(A, rows, W, out, offsets, counts_host, E, H, I, 2 * I, true, status,
                     ctx->num_sms, s);
  return gemm_call(A, rows, W, out, offsets, counts_host, E, I, H, H, false, status,
                   ctx->num_sms, s);
}

moe_status_t moe_grouped_gateup(const void* X, int64_t rows, int32_t H, int32_t I, int32_t E,
                                const int32_t* expert_offsets, const int32_t* expert_counts_host,
                                const void* W_gate_up, void* Act, uint32_t* status, void* stream) {
  return grouped_common(X, rows, H, I, E, expert_offsets, expert_counts_host, W_gate_up, Act,
                        status, stream, true);
}

moe_status_t moe_grouped_down(const void* Act, int64_t rows, int32_t H, int32_t I, int32_t E,
                              const int32_t* expert_offsets, const int32_t* expert_counts_host,
                              const void* W_down, void* Y, uint32_t* status, void* stream) {
  return grouped_common(Act, rows, H, I, E, expert_offsets, expert_counts_host, W_down, Y, status,
                        stream, false);
}

moe_status_t moe_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lock(g_mu);
  for (auto& r : g_prof.pending) {
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.pending.clear();
  g_prof.tot = moe_profile_t{};
  g_prof.timeline.clear();
  g_prof.origin_set = false;
  g_prof.calls = 0;
  g_prof.on = on != 0;
  return MOE_OK;
}

// Folds the pending event pairs into the totals and the kept launch records.
static moe_status_t prof_collect() {
  if (g_prof.pending.empty()) return MOE_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  for (auto& r : g_prof.pending) {
    float ms = 0.f, t0 = 0.f, t1 = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess ||
        cudaEventElapsedTime(&t0, g_prof.origin, r.a) != cudaSuccess ||
        cudaEventElapsedTime(&t1, g_prof.origin, r.b) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_prof.tot.launches[r.kind] += 1;
    g_prof.tot.ms[r.kind] += ms;
    g_prof.tot.rows[r.kind] += r.rows;
    g_prof.tot.active_experts[r.kind] += r.active;
    g_prof.tot.kernels += r.kernels;
    if (g_prof.timeline.size() < kTimelineCap) {
      moe_launch_record_t t;
      t.kind = r.kind;
      t.stream = r.stream_id;
      t.call = r.call;
      t.rows = r.rows;
      t.start_ms = t0;
      t.end_ms = t1;
      g_prof.timeline.push_back(t);
    }
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.pending.clear();
  return MOE_OK;
}

moe_status_t moe_profile_read(moe_profile_t* out) {
  if (!out) return MOE_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  moe_status_t st = prof_collect();
  if (st != MOE_OK) return st;
  *out = g_prof.tot;
  return MOE_OK;
}

moe_status_t moe_profile_timeline(moe_launch_record_t* records, int32_t capacity,
                                  int32_t* count) {
  if (!count || capacity < 0 || (capacity > 0 && !records)) return MOE_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  moe_status_t st = prof_collect();
  if (st != MOE_OK) return st;
  const size_t n = g_prof.timeline.size();
  const size_t m = n < (size_t)capacity ? n : (size_t)capacity;
  if (m) memcpy(records, g_prof.timeline.data(), sizeof(moe_launch_record_t) * m);
  *count = (int32_t)n;
  return MOE_OK;
}

}  // extern "C"
