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

// Build-time tuning knobs (the defaults are the shipped configuration).
#ifndef MOE_GEMM_2SM
// Which GEMMs run on CTA pairs (tcgen05 cta_group::2, 256-row tiles, M=128 across the pair
// for a tile of at most 128 rows) instead of single CTAs: bit 0 gate/up with TMA-loaded
// rows, bit 1 down, bit 2 gate/up with gathered rows (0: none, 7: all).
#define MOE_GEMM_2SM 0
#endif
#ifndef MOE_GEMM_BK
#define MOE_GEMM_BK 64  // K per stage: 64 (128-byte swizzle rows) or 32 (64-byte swizzle rows)
#endif
#ifndef MOE_GEMM_STAGES
#define MOE_GEMM_STAGES (MOE_GEMM_BK == 64 ? 4 : 8)  // single-CTA ring depth
#endif
#ifndef MOE_GEMM_STAGES_2SM
#define MOE_GEMM_STAGES_2SM (MOE_GEMM_BK == 64 ? 6 : 12)  // CTA-pair ring depth
#endif
#ifndef MOE_GEMM_L2_PROMO
#define MOE_GEMM_L2_PROMO 2  // TMA L2 promotion: 0 none, 1 128 B, 2 256 B
#endif
#ifndef MOE_GEMM_ORDER
#define MOE_GEMM_ORDER 0  // tile order inside an expert: 0 M tile fastest, 1 N tile fastest
#endif
#ifndef MOE_GEMM_EPI_STAGE
#define MOE_GEMM_EPI_STAGE 1  // 1: stage output blocks in shared memory for coalesced stores
#endif
#ifndef MOE_GEMM_DOWN_POLICY
#define MOE_GEMM_DOWN_POLICY 2  // L2 policy of the down GEMM's weights (same codes as below)
#endif
#ifndef MOE_GEMM_BAND
#define MOE_GEMM_BAND 16  // M tiles per raster band: an expert's A rows stay in L2 across N tiles
#endif
#ifndef MOE_GEMM_GATHER_MODE
#define MOE_GEMM_GATHER_MODE 0  // gathered A: 0 every warp a slice of every slot, 1 a slot per warp
#endif
#ifndef MOE_GEMM_HALF_TAILS
#define MOE_GEMM_HALF_TAILS 1  // a 128-row tile with at most 64 valid rows runs M=64 MMAs
#endif
#ifndef MOE_GEMM_GATHER_B_POLICY
#define MOE_GEMM_GATHER_B_POLICY 2  // gathered-A kernel: L2 policy of the weight loads
#endif
#ifndef MOE_GEMM_GATHER_A_POLICY
#define MOE_GEMM_GATHER_A_POLICY 0  // gathered-A kernel: 0 no hint, else L2 policy of the rows
#endif
#ifndef MOE_GEMM_TWO_M
#define MOE_GEMM_TWO_M 0  // 256-row tiles of two 128-row sub-tiles: bit 0 gate/up, bit 1 down
#endif
#ifndef MOE_GEMM_GATHER_DEPTH_2SM
#define MOE_GEMM_GATHER_DEPTH_2SM 2  // CTA pair, gathered A: stages of copies run ahead
#endif
#ifndef MOE_GEMM_GATHER_ARRIVE
// Single-CTA gathered A: 1 -- each gathering thread's copies of a stage arrive on its full
// barrier by themselves when they land (cp.async.mbarrier.arrive), so a stage is reported
// full as soon as its rows are in and the MMAs may run the whole ring ahead; 0 -- the
// threads wait for their oldest stage while they run ahead and arrive once per warp, which
// ties the MMAs of stage s to those of stage s - 2.
#define MOE_GEMM_GATHER_ARRIVE 1
#endif
#ifndef MOE_GEMM_DOWN_LSU
// 1: the down GEMM's A rows (Act, contiguous) are copied by the gathering warps with cp.async
// (through the SM's load path) instead of TMA, beside the weights' TMA loads
#define MOE_GEMM_DOWN_LSU 0
#endif
#ifndef MOE_GEMM_B_POLICY
#define MOE_GEMM_B_POLICY 2  // L2 policy of weight loads: 0 normal, 1 evict_first, 2 evict_last
#endif

namespace moe {
namespace {

constexpr int BN = kGemmBN, BK = MOE_GEMM_BK;
static_assert(BK == 64 || BK == 32, "K block of 64 (128-byte swizzle) or 32 (64-byte swizzle)");
constexpr uint32_t kSwizzleBytes = BK * 2;  // one swizzled row = the K block of one matrix row
constexpr int kRowsPerCta = 128;            // accumulator rows per CTA (TMEM lanes)
constexpr uint32_t kTmemCols = 2 * BN;      // two accumulators of BN fp32 columns
constexpr int kMaxE = 1024;

#ifndef MOE_GEMM_EPI_WARPS_2M
#define MOE_GEMM_EPI_WARPS_2M 8  // epilogue warps of the two-sub-tile kernel: 4 or 8
#endif
#ifndef MOE_GEMM_STAGES_2M
#define MOE_GEMM_STAGES_2M 3  // ring depth of the two-sub-tile kernel (64 KB stages)
#endif

// Geometry of one variant: single CTA with one 128-row A tile (128x256 tiles), single CTA
// with two 128-row A sub-tiles sharing each B tile (kTwoM, 256x256 tiles: two TMEM
// accumulators, one per sub-tile), or CTA pair (256x256 tiles, each CTA staging its 128 A
// rows and half of the 256 B rows).
template <bool kPair, bool kTwoM = false>
struct Geo {
  static_assert(!(kPair && kTwoM), "two sub-tiles per CTA are a single-CTA variant");
  static constexpr int kSubM = kTwoM ? 2 : 1;  // 128-row A sub-tiles staged per CTA
  static constexpr int kTileM = kPair ? 2 * kRowsPerCta : kSubM * kRowsPerCta;
  static constexpr int kStages =
      kPair ? MOE_GEMM_STAGES_2SM : (kTwoM ? MOE_GEMM_STAGES_2M : MOE_GEMM_STAGES);
  static constexpr uint32_t kABytes = kRowsPerCta * BK * 2;                 // 16 KB
  static constexpr uint32_t kAStageBytes = kSubM * kABytes;                 // 16 or 32 KB
  static constexpr uint32_t kBRows = kPair ? BN / 2 : BN;                   // B rows per CTA
  static constexpr uint32_t kBBytes = kBRows * BK * 2;                      // 16 or 32 KB
  static constexpr uint32_t kStageBytes = kAStageBytes + kBBytes;           // per CTA
  static constexpr uint32_t kTxBytes = kPair ? 2 * kStageBytes : kStageBytes;  // per stage
  static constexpr uint32_t kIdesc = umma_idesc_bf16_f32(kPair ? 2 * kRowsPerCta : kRowsPerCta, BN);
  // single CTA, one sub-tile: a tile holding at most 64 rows of its expert runs M=64 MMAs
  // (the accumulator's row r then sits in TMEM lane 32 (r / 16) + r % 16)
  // CTA pair: a tile holding at most 128 rows of its expert runs M=128 MMAs across the pair
  // (64 rows per CTA; each CTA's accumulator then holds tile columns 0..127 in TMEM lanes
  // 0..63 and columns 128..255 in lanes 64..127, 128 TMEM columns wide)
  static constexpr bool kHalfTails = !kTwoM && MOE_GEMM_HALF_TAILS != 0;
  static constexpr int kHalfRows = kPair ? kRowsPerCta : kRowsPerCta / 2;  // rows of a half tile
  static constexpr uint32_t kIdescHalf = umma_idesc_bf16_f32(kPair ? kRowsPerCta : kRowsPerCta / 2, BN);
  // bytes one stage of a pair's half tile brings to the leader's barrier (both CTAs)
  static constexpr uint32_t kTxBytesHalf = 2 * (kABytes / 2 + kBBytes);
  // epilogue warps: kTwoM may use two per TMEM lane quarter (each takes half the columns)
  static constexpr int kEpiWarps = kTwoM ? MOE_GEMM_EPI_WARPS_2M : 4;
};

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
  int32_t total_tiles;  // -1: count them here from the offsets (skipped on a bad index)
  const int32_t* gather;  // gathered A: token row of each permuted row (nullptr: plain A,
                          // or in the gathered kernel row r itself: A copied by the gathering
                          // warps instead of TMA)
  const uint8_t* gsrc;    // gathered A: the token rows (hidden), and their stride in bytes
  int64_t gsrc_stride;
  int32_t K;              // valid K columns (gathered A: the rest of the last block reads 0)
  int64_t gsrc_rows;  // checks build: rows of the gathered source
  int64_t out_rows;   // checks build: rows of out
};

template <int kStages>
struct SmemCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Threads of one CTA: producer, MMA, the epilogue warps; + 4 gathering warps (gathered A).
template <bool kGather, bool kTwoM = false>
__host__ __device__ constexpr int gemm_threads() {
  return 64 + 32 * Geo<false, kTwoM>::kEpiWarps + (kGather ? kGatherThreads : 0);
}
static_assert(gemm_threads<false>() == kGemmThreads, "thread layout");

constexpr size_t kCtlBytes = 256;
static_assert(sizeof(SmemCtl<MOE_GEMM_STAGES_2SM>) <= kCtlBytes, "control block");
static_assert(sizeof(SmemCtl<MOE_GEMM_STAGES>) <= kCtlBytes, "control block");

// Epilogue staging: per epilogue warp one block of 32 rows x 32 bf16 columns, rows padded
// to 80 bytes so that both the row-wise writes and the 8-rows-per-instruction reads are
// free of bank conflicts within each 8-lane phase.
constexpr int kEpiRowBytes = 80;
constexpr int kEpiWarpBytes = 32 * kEpiRowBytes;
constexpr size_t kTablesBytes = (2 * (kMaxE + 1) * sizeof(int32_t) + 15) & ~size_t(15);

template <bool kPair, bool kTwoM = false>
constexpr size_t smem_bytes() {
  using G = Geo<kPair, kTwoM>;
  return 1024 /*alignment slack*/ + G::kStages * G::kStageBytes + kCtlBytes + kTablesBytes +
         (MOE_GEMM_EPI_STAGE ? G::kEpiWarps * kEpiWarpBytes : 0);
}
static_assert(smem_bytes<false, true>() <= 232448, "two-sub-tile kernel exceeds 227 KB");
static_assert(sizeof(SmemCtl<MOE_GEMM_STAGES_2M>) <= kCtlBytes, "control block");

// A tile: expert e, column tile n, row tile m of the expert's rows.
struct Tile {
  int32_t e, n, m;
};

__device__ uint32_t g_range_flags;  // checks build: a row index outside its buffer was seen

template <int kTileM>
__device__ __forceinline__ Tile decode_tile(int32_t L, const int32_t* tile_start,
                                            const int32_t* off, int32_t E, int32_t n_tiles) {
  // largest e with tile_start[e] <= L; that expert has at least one tile
  int32_t lo = 0, hi = E - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= L) lo = mid;
    else hi = mid - 1;
  }
  const int32_t mt = (off[lo + 1] - off[lo] + kTileM - 1) / kTileM;
  const int32_t local = L - tile_start[lo];
  Tile t;
  t.e = lo;
#if MOE_GEMM_ORDER == 0
  // bands of up to MOE_GEMM_BAND M tiles; inside a band M is fastest, then N
  const int32_t band_tiles = MOE_GEMM_BAND * n_tiles;
  const int32_t b = local / band_tiles;
  const int32_t inner = local - b * band_tiles;
  const int32_t width = min(MOE_GEMM_BAND, mt - b * MOE_GEMM_BAND);
  t.n = inner / width;
  t.m = b * MOE_GEMM_BAND + (inner - t.n * width);
#else
  t.m = local / n_tiles;
  t.n = local - t.m * n_tiles;
#endif
  return t;
}

// Stores the 32 x 32 bf16 block of one epilogue warp: lane i holds row (32 q + i) of the
// tile as 16 packed bf16 pairs.  Rows at or past rows_valid (past the expert's end) and
// columns at or past out_cols are never written.
// kRpw: rows per warp, 32 (M=128 accumulator: lane i of quarter q is tile row 32 q + i) or
// 16 (M=64 accumulator: lanes 0..15 of quarter q hold tile rows 16 q + i, lanes 16..31
// nothing).
__device__ __forceinline__ void store_block(const uint32_t (&packed)[16], uint8_t* wbuf, int lane,
                                            int q, bool row_ok, int32_t rows_valid,
                                            int64_t row_base, int32_t col0, const KParams& p,
                                            __nv_bfloat16* out, int64_t out_rows,
                                            int rpw = 32) {
#if MOE_GEMM_EPI_STAGE
  uint4* mine = reinterpret_cast<uint4*>(wbuf + lane * kEpiRowBytes);
#pragma unroll
  for (int v = 0; v < 4; ++v)
    mine[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
  __syncwarp();
  // 8 rows x 64 contiguous bytes per instruction: lane = 4 * (row % 8) + 16-byte segment
  const int seg = lane & 3;
  const int32_t col = col0 + seg * 8;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int rr = pass * 8 + (lane >> 2);
    if (pass * 8 >= rpw) break;
    const uint4 v = *reinterpret_cast<const uint4*>(wbuf + rr * kEpiRowBytes + seg * 16);
    const int32_t tr = q * rpw + rr;  // row inside the CTA's 128 rows
    if (tr < rows_valid && col < p.out_cols &&
        check_row(row_base + tr, out_rows, &g_range_flags))
      *reinterpret_cast<uint4*>(out + (row_base + tr) * p.out_cols + col) = v;
  }
  __syncwarp();
  (void)row_ok;
#else
  (void)wbuf;
  (void)rows_valid;
  if (row_ok && check_row(row_base + q * rpw + lane, out_rows, &g_range_flags)) {
    uint4* dst = reinterpret_cast<uint4*>(out + (row_base + q * rpw + lane) * p.out_cols + col0);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      if (col0 + v * 8 < p.out_cols)
        dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
  }
#endif
}

// One persistent CTA (kPair = false) or CTA pair (kPair = true, cluster of 2) per tile
// stream.  In a pair, the even CTA ("leader") owns the full-stage barriers and the MMA
// issue; both CTAs load their own halves, run their own epilogue on their own TMEM rows,
// and report back to the leader.  A pair's tile of at most 128 rows of its expert runs
// M=128 MMAs (64 rows per CTA, loaded as 64-row boxes); with gathered A rows each CTA's
// gathering warps copy its own rows and arrive on the leader's barrier.
//
// kTwoM (single CTA): a tile is 256 rows of one expert by one N tile, staged as two 128-row
// A sub-tiles that share every B stage, each with its own 128 x 256 TMEM accumulator (the
// two fill all 512 columns).  Per 64-wide K block the CTA loads 64 KB for twice the MMAs of
// a 48 KB one-sub-tile stage, so the same shared memory holds 1.5x the MMA time in flight
// and each SM pulls 2/3 of the bytes per flop.  A tile whose expert ends within its first
// 128 rows has no second sub-tile (no load, no MMA, no epilogue).  With no second
// accumulator to alternate with, the MMA warp starts a tile's first-sub-tile MMAs as soon
// as the epilogue has read that accumulator, and holds back (up to kStages - 1 stages) the
// second sub-tile's MMAs until the epilogue has read the other one.
// tmA64 / tmB64: the same matrices with 64-row boxes (the CTA pair's half tiles).
template <bool kSwiGLU, bool kPair, bool kGather, bool kTwoM>
__device__ __forceinline__ void gemm_body(const CUtensorMap* tmA, const CUtensorMap* tmB,
                                          const CUtensorMap* tmA64, const CUtensorMap* tmB64,
                                          const KParams& p) {
  using G = Geo<kPair, kTwoM>;
  constexpr int STAGES = G::kStages;
  constexpr int kEpiWarps = G::kEpiWarps;
  constexpr int kFirstGatherWarp = 2 + kEpiWarps;
  // Gathering threads keep kGatherDepth + 1 stages of copies in flight and arrive on a
  // stage's full barrier only once they have issued the copies of the kGatherDepth stages
  // after it, so those stages must be free (released by the MMA warp) by then: the MMAs of
  // stage s wait for those of stage s + kGatherDepth - STAGES.
  constexpr int kGatherDepth =
      kPair ? MOE_GEMM_GATHER_DEPTH_2SM : (STAGES - 2 > 0 ? STAGES - 2 : 1);
  // kTwoM: stages whose second-sub-tile MMAs the MMA warp may hold back (each held stage
  // stays unreleased); with gathered A the gathering threads' run-ahead must stay free.
  constexpr int kMaxHeld = STAGES - 1 - (kGather ? kGatherDepth : 0);
  // Gathered A, one ring slot per gathering warp (the single-sub-tile ring of 4 slots)
  constexpr bool kWarpStages =
      kGather && !kTwoM && MOE_GEMM_GATHER_MODE == 1 && STAGES == kGatherThreads / 32;
  // Gathered A arriving through the copies themselves (single CTA; a pair's full barrier
  // belongs to the other CTA)
  constexpr bool kCopyArrive = kGather && !kPair && !kWarpStages && MOE_GEMM_GATHER_ARRIVE != 0;
  static_assert(!kTwoM || kMaxHeld >= 0, "ring too shallow for the gathered two-sub-tile kernel");
  static_assert(!(kWarpStages && kPair), "one ring slot per gathering warp: single CTAs only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * G::kAStageBytes;
  SmemCtl<STAGES>* ctl = reinterpret_cast<SmemCtl<STAGES>*>(smem + STAGES * G::kStageBytes);
  int32_t* off = reinterpret_cast<int32_t*>(smem + STAGES * G::kStageBytes + kCtlBytes);
  int32_t* tile_start = off + (kMaxE + 1);
  uint8_t* epi_stage = smem + STAGES * G::kStageBytes + kCtlBytes + kTablesBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t E = p.E;
  const uint32_t rank = kPair ? cluster_cta_rank() : 0;
  const bool leader = rank == 0;
  const int32_t stream_id = kPair ? (int32_t)(blockIdx.x >> 1) : (int32_t)blockIdx.x;
  const int32_t n_streams = kPair ? (int32_t)(gridDim.x >> 1) : (int32_t)gridDim.x;

  // ---- set-up: expert offsets, tile prefix, barriers, TMEM ----
  for (int32_t i = threadIdx.x; i <= E; i += blockDim.x) off[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // gathered A: the weight producer's arrival plus one per A-gathering warp (or one per
      // slot-owning gathering warp); CTA pair: both CTAs' gathering warps arrive on the
      // leader's barrier
      mbar_init(&ctl->full[s],
                kGather ? 1 + (kWarpStages ? 1
                               : kCopyArrive ? kGatherThreads
                                             : (kPair ? 2 : 1) * (kGatherThreads / 32))
                        : 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tfull[b], 1);
      mbar_init(&ctl->tempty[b], (kPair ? 2 : 1) * kEpiWarps * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(tmB);
    if (kPair) {
      tma_prefetch_desc(tmA64);
      tma_prefetch_desc(tmB64);
    }
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&ctl->tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
  __syncthreads();
  if (warp == 2) {
    // exclusive prefix of tiles per expert: lane l covers experts [l*per, (l+1)*per)
    const int32_t per = (E + 31) / 32;
    const int32_t e0 = lane * per, e1 = min(E, e0 + per);
    int32_t sum = 0;
    auto tiles_of = [&](int32_t e) {
      return (off[e + 1] - off[e] + G::kTileM - 1) / G::kTileM * p.n_tiles;
    };
    for (int32_t e = e0; e < e1; ++e) sum += tiles_of(e);
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int32_t run = incl - sum;
    for (int32_t e = e0; e < e1; ++e) {
      tile_start[e] = run;
      run += tiles_of(e);
    }
    if (lane == 31) tile_start[E] = incl;
  }
  tc_fence_before();
  if (kPair) cluster_sync();  // the peer's loads target the leader's barriers: init first
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int* abort = &ctl->abort;
  // Tiles of the launch: given by the host, or (total_tiles < 0: the host has not seen the
  // counts) the prefix over the experts -- none when the metadata of this call flagged an
  // expert index out of range, whose offsets are then not to be used.
  const int32_t total = p.total_tiles >= 0 ? p.total_tiles
                        : (*reinterpret_cast<volatile uint32_t*>(p.status) & MOE_DEV_BAD_INDEX)
                            ? 0
                            : tile_start[E];

  // kTwoM: whether tile t has a second 128-row sub-tile (its expert has rows past the first)
  auto has_m1 = [&](const Tile& t) {
    return kTwoM && off[t.e + 1] - off[t.e] > t.m * G::kTileM + kRowsPerCta;
  };
  // kHalfTails: whether tile t holds at most kHalfRows rows of its expert (single CTA: M=64
  // MMAs; pair: M=128 MMAs, 64 rows per CTA)
  auto is_half = [&](const Tile& t) {
    return G::kHalfTails && off[t.e + 1] - off[t.e] - t.m * G::kTileM <= G::kHalfRows;
  };
  // first tile row this CTA stages (pair: CTA 1 takes the second 128 rows, or of a half tile
  // the second 64)
  auto cta_row = [&](bool half) {
    return kPair ? (int32_t)rank * (half ? kRowsPerCta / 2 : kRowsPerCta) : 0;
  };
  // B rows of tile t this CTA stages (pair: CTA 0 the gate rows of the 128-column tile and
  // CTA 1 the up rows; of a gate/up half tile each CTA 64 gate rows and the same 64 up rows,
  // so that the columns of one lane half pair gate with up)
  auto stage_b = [&](const Tile& t, bool half, uint8_t* b_dst, uint32_t bar, int32_t kb,
                     uint64_t pol) {
    if (!kPair) return;
    if (kSwiGLU && half) {
      const int32_t g0 = t.e * p.b_rows + t.n * (BN / 2) + (int32_t)rank * (BN / 4);
      tma_load_2d_pair(b_dst, tmB64, bar, kb * BK, g0, pol);
      tma_load_2d_pair(b_dst + G::kBBytes / 2, tmB64, bar, kb * BK, g0 + p.up_off, pol);
    } else {
      const int32_t brow = kSwiGLU ? t.e * p.b_rows + t.n * (BN / 2) + (int32_t)rank * p.up_off
                                   : t.e * p.b_rows + t.n * BN + (int32_t)rank * (BN / 2);
      tma_load_2d_pair(b_dst, tmB, bar, kb * BK, brow, pol);
    }
  };

  if (warp == 0 && kGather) {
    // ---------------- weight producer, gathered A (lane 0) ----------------
    // The A rows of a stage come from the gathering warps (below); this lane arms the stage
    // with the weight bytes and loads the weight box(es) with TMA.
    if (lane == 0) {
      const uint64_t pol_w = MOE_GEMM_GATHER_B_POLICY == 1   ? l2_policy_evict_first()
                             : MOE_GEMM_GATHER_B_POLICY == 2 ? l2_policy_evict_last()
                                                             : l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int32_t L = stream_id; L < total && ok; L += n_streams) {
        const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
        const int32_t brow = t.e * p.b_rows + t.n * (kSwiGLU ? BN / 2 : BN);
        const bool half = is_half(t);
        for (int32_t kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          uint8_t* b_dst = sB + stage * G::kBBytes;
          if (kPair) {
            // both CTAs' weight halves count on the leader's barrier
            if (leader) mbar_arrive_expect_tx(&ctl->full[stage], 2 * G::kBBytes);
            stage_b(t, half, b_dst, mapa_shared(smem_u32(&ctl->full[stage]), 0), kb, pol_w);
          } else {
            mbar_arrive_expect_tx(&ctl->full[stage], G::kBBytes);
            tma_load_2d(b_dst, tmB, &ctl->full[stage], kb * BK, brow, pol_w);
            if (kSwiGLU)
              tma_load_2d(b_dst + G::kBBytes / 2, tmB, &ctl->full[stage], kb * BK,
                          brow + p.up_off, pol_w);
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader)
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_drain(&ctl->full[s], (armed_parity >> s) & 1u, 100000000ull);
    }
  } else if (kGather && kWarpStages && warp >= kFirstGatherWarp) {
    // ---------------- A producers, gathered rows, one ring slot per warp ----------------
    // Gathering warp w fills ring slot w (the ring has as many slots as there are gathering
    // warps): for each K block that lands in slot w it copies all of the tile's A rows --
    // lane (8 s + j) copies 16-byte chunk j of rows 4 i + s, i < 32 -- into the
    // 128-byte-swizzled K-major layout, waits for its own copies, makes them visible to the
    // async proxy, and one lane arrives on the slot's full barrier.  A slot is thus reported
    // full as soon as its copies have landed, and each slot's copies are in flight for up to
    // a whole lap of the ring.  Lane l holds the token indices of rows l, l+32, l+64, l+96.
    const int gw = warp - kFirstGatherWarp, j = lane & 7, sub = lane >> 3;
    const uint64_t pol_a = MOE_GEMM_GATHER_A_POLICY == 1 ? l2_policy_evict_first()
                           : MOE_GEMM_GATHER_A_POLICY == 2 ? l2_policy_evict_last()
                                                           : l2_policy_evict_normal();
    const int32_t* gat = p.gather;
    auto load_tokens = [&](int32_t L2, int32_t (&tok)[4]) {
      const Tile t2 = decode_tile<G::kTileM>(L2, tile_start, off, E, p.n_tiles);
      const int32_t row0 = off[t2.e] + t2.m * G::kTileM;
      const int32_t last = off[t2.e + 1] - 1;  // rows past the expert re-read its last row
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int32_t r = min(row0 + q * 32 + lane, last);
        tok[q] = gat ? gat[r] : r;
      }
    };
    int32_t next_tok[4];
    if (stream_id < total) load_tokens(stream_id, next_tok);
    uint32_t phase = 0;  // phase of this warp's slot
    int32_t sigma = 0;   // K blocks of this CTA so far (ring position)
    bool ok = true;
    for (int32_t L = stream_id; L < total && ok; L += n_streams) {
      const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
      const bool half = is_half(t);  // M=64 MMAs read rows 0..63 only
      int32_t tok[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        tok[q] = next_tok[q];
        if (!check_row(tok[q], p.gsrc_rows, &g_range_flags)) tok[q] = 0;
      }
      if (L + n_streams < total) load_tokens(L + n_streams, next_tok);
      for (int32_t kb = 0; kb < p.num_kb; ++kb, ++sigma) {
        if ((sigma & (STAGES - 1)) != gw) continue;
        if (!__all_sync(0xffffffffu, mbar_wait(&ctl->empty[gw], phase ^ 1u, abort, p.status))) {
          ok = false;
          break;
        }
        const uint32_t a = smem_u32(sA + gw * G::kAStageBytes);
        const uint32_t nbytes = (kb * BK + j * 8 < p.K) ? 16u : 0u;  // zero past K
        const uint8_t* base = p.gsrc + j * 16 + kb * (BK * 2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (half && i >= 16) break;
          const int32_t r = 4 * i + sub;
          const int64_t tk = __shfl_sync(0xffffffffu, tok[i / 8], 4 * (i % 8) + sub);
          const uint32_t dst_s = a + r * (BK * 2) + ((j ^ (r & 7)) << 4);
          if (MOE_GEMM_GATHER_A_POLICY == 0)
            cp_async_16(dst_s, base + tk * p.gsrc_stride, nbytes);
          else
            cp_async_16_hint(dst_s, base + tk * p.gsrc_stride, nbytes, pol_a);
        }
        cp_async_commit();
        cp_async_wait<0>();
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->full[gw]);
        phase ^= 1u;
      }
    }
    (void)ok;
  } else if (kGather && warp >= kFirstGatherWarp) {
    // ---------------- A producers, gathered rows (4 warps, LSU) ----------------
    // The tile's A rows are the token rows src_tok[row] of `hidden`.  Per K block, lane
    // (8 s + j) of gathering warp w copies 16-byte chunk j of rows 32 w + 4 i + s (i < 8) of
    // each 128-row sub-tile with cp.async, into the 128-byte-swizzled K-major layout the MMA
    // reads (chunk j of row r at position j ^ (r % 8)); a warp instruction covers 4 whole
    // 128-byte row segments.  A thread keeps kDepth + 1 stages of copies in flight; when
    // its oldest stage has landed it makes the writes visible to the async proxy, and once
    // every lane of the warp has, one lane arrives on that stage's full barrier (one arrival
    // per warp: for a CTA pair the arrivals cross to the other SM, and 128 per stage from
    // each CTA would cost more than the copies).
    constexpr int kDepth = kGatherDepth;
    constexpr int kSub = G::kSubM;
    const int gw = warp - kFirstGatherWarp, j = lane & 7, sub = lane >> 3;
    const uint64_t pol_a = MOE_GEMM_GATHER_A_POLICY == 1 ? l2_policy_evict_first()
                           : MOE_GEMM_GATHER_A_POLICY == 2 ? l2_policy_evict_last()
                                                           : l2_policy_evict_normal();
    int stage = 0;
    uint32_t phase = 0;
    int32_t issued = 0, arrived = 0;
    bool ok = true;
    const int32_t* gat = p.gather;  // gathered A has one row segment
    // (every wait's outcome is made warp-uniform, so that the lanes leave the loop together
    // and the per-warp arrivals below never wait on a lane that has gone)
    // token index of each row this thread copies in tile L (rows past the expert re-read
    // its last row)
    auto load_tokens = [&](int32_t L2, int32_t (&tok)[kSub * 8]) {
      const Tile t2 = decode_tile<G::kTileM>(L2, tile_start, off, E, p.n_tiles);
      const int32_t row0 = off[t2.e] + t2.m * G::kTileM + cta_row(is_half(t2));
      const int32_t last = off[t2.e + 1] - 1;
#pragma unroll
      for (int h = 0; h < kSub; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int32_t r = min(row0 + h * kRowsPerCta + gw * 32 + 4 * i + sub, last);
          tok[h * 8 + i] = gat ? gat[r] : r;
        }
    };
    // the next tile's indices are loaded when a tile starts, so that their latency is
    // spent behind the tile's copies instead of at the next tile boundary
    int32_t next_tok[kSub * 8];
    if (stream_id < total) load_tokens(stream_id, next_tok);
    // a stage's full barrier (the leader's, for a CTA pair: its MMAs read both CTAs' rows),
    // once per warp after every lane's copies of the stage are visible to the async proxy
    // (CTA pair: released at CTA scope like the other arrivals of a pair on the leader's
    // barriers -- at cluster scope the release waits for every copy the thread still has in
    // flight, ~2000 cycles per stage)
    auto arrive_full = [&](int s) {
      __syncwarp();
      if (lane == 0) {
        if (kPair) mbar_arrive_remote(mapa_shared(smem_u32(&ctl->full[s]), 0));
        else mbar_arrive(&ctl->full[s]);
      }
    };
    for (int32_t L = stream_id; L < total && ok; L += n_streams) {
      const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
      const int n_sub = has_m1(t) ? 2 : 1;
      // half tiles: only rows 0..63 are read by the M=64 MMAs (gathering warps 0 and 1)
      const bool skip = is_half(t) && gw >= 2;
      const uint8_t* src[kSub * 8];
#pragma unroll
      for (int x = 0; x < kSub * 8; ++x) {
        int64_t tok = next_tok[x];
        if (!check_row(tok, p.gsrc_rows, &g_range_flags)) tok = 0;
        src[x] = p.gsrc + tok * p.gsrc_stride + j * 16;
      }
      if (L + n_streams < total) load_tokens(L + n_streams, next_tok);
      for (int32_t kb = 0; kb < p.num_kb; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&ctl->empty[stage], phase ^ 1u, abort, p.status))) {
          ok = false;
          break;
        }
        const uint32_t a = smem_u32(sA + stage * G::kAStageBytes);
        const uint32_t nbytes = (kb * BK + j * 8 < p.K) ? 16u : 0u;  // zero past K
#pragma unroll
        for (int h = 0; h < kSub; ++h) {
          if (h < n_sub && !skip) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int32_t r = gw * 32 + 4 * i + sub;
              const uint32_t dst_s = a + h * G::kABytes + r * (BK * 2) + ((j ^ (r & 7)) << 4);
              if (MOE_GEMM_GATHER_A_POLICY == 0)
                cp_async_16(dst_s, src[h * 8 + i] + kb * (BK * 2), nbytes);
              else
                cp_async_16_hint(dst_s, src[h * 8 + i] + kb * (BK * 2), nbytes, pol_a);
            }
          }
        }
        if (kCopyArrive) {
          cp_async_arrive_noinc(&ctl->full[stage]);
        } else {
          cp_async_commit();
          ++issued;
          if (issued - arrived > kDepth) {
            cp_async_wait<kDepth>();
            fence_async_smem();
            arrive_full(arrived % STAGES);
            ++arrived;
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    cp_async_wait<0>();
    fence_async_smem();
    if (!kCopyArrive)
      for (; arrived < issued; ++arrived) arrive_full(arrived % STAGES);
    (void)ok;
  } else if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      const int pol_code = kSwiGLU ? MOE_GEMM_B_POLICY : MOE_GEMM_DOWN_POLICY;
      const uint64_t pol_w = pol_code == 1   ? l2_policy_evict_first()
                             : pol_code == 2 ? l2_policy_evict_last()
                                             : l2_policy_evict_normal();
      const uint64_t pol_a = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bits, for the abort drain
      bool ok = true;
      for (int32_t L = stream_id; L < total && ok; L += n_streams) {
        // A row and B row of tile L (of this CTA's tile stream)
        const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
        const bool half = kPair && is_half(t);
        const int32_t row0 = off[t.e] + t.m * G::kTileM + cta_row(half);
        const int32_t brow = t.e * p.b_rows + t.n * (kSwiGLU ? BN / 2 : BN);  // single CTA
        const bool m1 = has_m1(t);
        const uint32_t tx = kTwoM ? (m1 ? G::kStageBytes : G::kABytes + G::kBBytes) : G::kTxBytes;
        const CUtensorMap* mapA = tmA;
        for (int32_t kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = sA + stage * G::kAStageBytes;
          uint8_t* b_dst = sB + stage * G::kBBytes;
          if (kPair) {
            if (leader)
              mbar_arrive_expect_tx(&ctl->full[stage], half ? G::kTxBytesHalf : G::kTxBytes);
            const uint32_t bar = mapa_shared(smem_u32(&ctl->full[stage]), 0);
            tma_load_2d_pair(a_dst, half ? tmA64 : mapA, bar, kb * BK, row0, pol_a);
            stage_b(t, half, b_dst, bar, kb, pol_w);
          } else {
            mbar_arrive_expect_tx(&ctl->full[stage], tx);
            tma_load_2d(a_dst, mapA, &ctl->full[stage], kb * BK, row0, pol_a);
            if (kTwoM && m1)
              tma_load_2d(a_dst + G::kABytes, mapA, &ctl->full[stage], kb * BK,
                          row0 + kRowsPerCta, pol_a);
            if (kSwiGLU) {
              tma_load_2d(b_dst, tmB, &ctl->full[stage], kb * BK, brow, pol_w);
              tma_load_2d(b_dst + G::kBBytes / 2, tmB, &ctl->full[stage], kb * BK,
                          brow + p.up_off, pol_w);
            } else {
              tma_load_2d(b_dst, tmB, &ctl->full[stage], kb * BK, brow, pol_w);
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
      if (!ok && leader) {
        // wait (bounded) for the copies already issued, so none lands after exit
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_drain(&ctl->full[s], (armed_parity >> s) & 1u, 100000000ull);
      }
    }
  } else if (warp == 1 && kTwoM) {
    // ---------------- MMA issuer, two sub-tiles per tile ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t use[2] = {0, 0};  // tiles that used accumulator 0 / 1 so far
      bool ok = true, issued = false;
      auto mma_sub = [&](int h, int st, int32_t kb) {
        const uint32_t a_addr = smem_u32(sA + st * G::kAStageBytes + h * G::kABytes);
        const uint32_t b_addr = smem_u32(sB + st * G::kBBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = kmajor_desc<kSwizzleBytes>(a_addr + kk * 32);
          const uint64_t bd = kmajor_desc<kSwizzleBytes>(b_addr + kk * 32);
          umma_bf16(tmem_base + h * BN, ad, bd, G::kIdesc, (kb | kk) != 0);
        }
      };
      for (int32_t L = stream_id; L < total && ok; L += n_streams) {
        const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
        const bool m1 = has_m1(t);
        if (!mbar_wait(&ctl->tempty[0], (use[0] & 1u) ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool acc1 = false;        // accumulator 1 read out by the epilogue, this tile
        int pend_stage[STAGES];   // stages whose second-sub-tile MMAs wait for accumulator 1
        int32_t pend_kb[STAGES];
        int npend = 0;
        for (int32_t kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, abort, p.status)) {
            ok = false;
            break;
          }
          if (kCopyArrive) fence_async_smem();
          tc_fence_after();
          mma_sub(0, stage, kb);
          issued = true;
          if (kb == p.num_kb - 1) umma_commit(&ctl->tfull[0]);
          if (m1) {
            if (!acc1) {
              acc1 = mbar_test_wait(&ctl->tempty[1], (use[1] & 1u) ^ 1u);
              if (!acc1 && (npend >= kMaxHeld || kb == p.num_kb - 1)) {
                if (!mbar_wait(&ctl->tempty[1], (use[1] & 1u) ^ 1u, abort, p.status)) {
                  ok = false;
                  break;
                }
                acc1 = true;
              }
              if (acc1) tc_fence_after();
            }
            if (acc1) {
              for (int i = 0; i < npend; ++i) {
                mma_sub(1, pend_stage[i], pend_kb[i]);
                umma_commit(&ctl->empty[pend_stage[i]]);
              }
              npend = 0;
              mma_sub(1, stage, kb);
              umma_commit(&ctl->empty[stage]);
            } else {
              pend_stage[npend] = stage;
              pend_kb[npend] = kb;
              ++npend;
            }
          } else {
            umma_commit(&ctl->empty[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ++use[0];
        if (m1) {
          umma_commit(&ctl->tfull[1]);
          ++use[1];
        }
      }
      if (!ok && issued) {
        // every MMA issued so far must finish before TMEM is released
        umma_commit(&ctl->drain);
        mbar_drain(&ctl->drain, 0, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (the leader only) ----------------
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      int32_t it = 0;
      for (int32_t L = stream_id; L < total && ok; L += n_streams, ++it) {
        const int buf = it & 1;
        const uint32_t tphase = (it >> 1) & 1;
        if (!mbar_wait(&ctl->tempty[buf], tphase ^ 1u, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        uint32_t idesc = G::kIdesc;
        if (G::kHalfTails) {
          const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
          if (is_half(t)) idesc = G::kIdescHalf;
        }
        for (int32_t kb = 0; kb < p.num_kb; ++kb) {
          // (pair with gathered rows: the other CTA's gathering threads released its rows)
          if (!mbar_wait(&ctl->full[stage], phase, abort, p.status)) {
            ok = false;
            break;
          }
          // copies that arrived by themselves wrote through the generic proxy: make them
          // visible to the MMAs' (async-proxy) reads
          if (kCopyArrive) fence_async_smem();
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * G::kAStageBytes);
          const uint32_t b_addr = smem_u32(sB + stage * G::kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // advance 16 bf16 = 32 bytes along K inside the swizzled row
            const uint64_t ad = kmajor_desc<kSwizzleBytes>(a_addr + kk * 32);
            const uint64_t bd = kmajor_desc<kSwizzleBytes>(b_addr + kk * 32);
            if (kPair) umma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0);
            else umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          issued = true;
          if (kPair) umma_commit_pair(&ctl->empty[stage], 0x3);
          else umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (kPair) umma_commit_pair(&ctl->tfull[buf], 0x3);
        else umma_commit(&ctl->tfull[buf]);
      }
      if (!ok && issued) {
        // every MMA issued so far must finish before TMEM is released
        if (kPair) umma_commit_pair(&ctl->drain, 0x1);
        else umma_commit(&ctl->drain);
        mbar_drain(&ctl->drain, 0, 100000000ull);
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // ---------------- epilogue (warps 2 .. 2 + kEpiWarps - 1 of both CTAs) ----------------
    // Warp w reads TMEM lanes 32 (w % 4) .. +31 (the lane quarter its SM sub-partition may
    // access).  kTwoM: two warps per quarter, each taking half of the column chunks; the
    // tile's accumulators are read one after the other (sub-tile 0, then 1).
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    constexpr int kParts = kEpiWarps / 4;  // warps sharing one lane quarter
    const int half = kParts > 1 ? (warp - 2) / 4 : 0;
    uint8_t* wbuf = epi_stage + (warp - 2) * kEpiWarpBytes;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&ctl->tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&ctl->tempty[1]), 0);
    uint32_t use[2] = {0, 0};
    int32_t it = 0;
    bool ok = true;
    for (int32_t L = stream_id; L < total && ok; L += n_streams, ++it) {
      const Tile t = decode_tile<G::kTileM>(L, tile_start, off, E, p.n_tiles);
      const int n_acc = has_m1(t) ? 2 : 1;
      for (int h = 0; h < n_acc; ++h) {
        // accumulator of this sub-tile: kTwoM h; otherwise alternating per tile
        const int buf = kTwoM ? h : (it & 1);
        const uint32_t tphase = kTwoM ? (use[h] & 1u) : ((it >> 1) & 1);
        if (!mbar_wait(&ctl->tfull[buf], tphase, abort, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int32_t* offs = off;
        __nv_bfloat16* out = p.out;
        const int64_t out_rows = p.out_rows;
        const bool hf = is_half(t);  // (`half` is the kTwoM column half of this warp)
        const int32_t first = t.m * G::kTileM + cta_row(hf) + h * kRowsPerCta;
        const int32_t rows_valid = offs[t.e + 1] - offs[t.e] - first;
        const int64_t row_base = (int64_t)offs[t.e] + first;  // output row of TMEM lane 0
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * BN;
        if (kPair && hf) {
          // M=128 across the pair: this CTA's 64 rows; lane quarter q holds rows
          // 32 (q % 2) .. +31 and tile columns 128 (q / 2) .. +127 in TMEM columns 0..127
          // (gate/up: gate columns 0..63 and the matching up columns 64..127)
          const int rq = q & 1, ch = q >> 1;
          const bool ok_row = rq * 32 + lane < rows_valid;
          constexpr int kHalfChunks = kSwiGLU ? 2 : 4;
#pragma unroll 1
          for (int c = 0; c < kHalfChunks; ++c) {
            uint32_t packed[16];
            int32_t col0;
            if (kSwiGLU) {
              uint32_t g[32], u[32];
              tmem_ld_32cols(t_row + c * 32, g);
              tmem_ld_32cols(t_row + 64 + c * 32, u);
              tmem_ld_wait2(g, u);
              col0 = t.n * (BN / 2) + ch * 64 + c * 32;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                const float a0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
                const float a1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
                packed[i] = pack_bf16x2(a0, a1);
              }
            } else {
              uint32_t acc[32];
              tmem_ld_32cols(t_row + c * 32, acc);
              tmem_ld_wait(acc);
              col0 = t.n * BN + ch * 128 + c * 32;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                packed[i] =
                    pack_bf16x2(__uint_as_float(acc[2 * i]), __uint_as_float(acc[2 * i + 1]));
            }
            store_block(packed, wbuf, lane, rq, ok_row, rows_valid, row_base, col0, p,
                        p.out, p.out_rows, 32);
          }
        } else if (kSwiGLU) {
          const int rpw = hf ? 16 : 32;  // M=64 accumulator: 16 rows per lane quarter
          const bool row_ok = rpw == 32 ? r < rows_valid : (lane < 16 && q * 16 + lane < rows_valid);
          constexpr int kChunks = (BN / 2) / 32 / kParts;
#pragma unroll 1
          for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
            uint32_t g[32], u[32];
            tmem_ld_32cols(t_row + c * 32, g);
            tmem_ld_32cols(t_row + BN / 2 + c * 32, u);
            tmem_ld_wait2(g, u);
            const int32_t col0 = t.n * (BN / 2) + c * 32;
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              // silu(g) = g / (1 + e^-g); the fast division (no IEEE slow path) is exact to a
              // few ulp, far below the bf16 rounding of the result
              const float a0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
              const float a1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
              packed[i] = pack_bf16x2(a0, a1);
            }
            store_block(packed, wbuf, lane, q, row_ok, rows_valid, row_base, col0, p, out,
                        out_rows, rpw);
          }
        } else {
          const int rpw = hf ? 16 : 32;
          const bool row_ok = rpw == 32 ? r < rows_valid : (lane < 16 && q * 16 + lane < rows_valid);
          constexpr int kChunks = BN / 32 / kParts;
#pragma unroll 1
          for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
            uint32_t acc[32];
            tmem_ld_32cols(t_row + c * 32, acc);
            tmem_ld_wait(acc);
            const int32_t col0 = t.n * BN + c * 32;
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] =
                  pack_bf16x2(__uint_as_float(acc[2 * i]), __uint_as_float(acc[2 * i + 1]));
            store_block(packed, wbuf, lane, q, row_ok, rows_valid, row_base, col0, p, out,
                        out_rows, rpw);
          }
        }
        tc_fence_before();
        if (kPair) mbar_arrive_remote(buf ? tempty_leader1 : tempty_leader0);
        else mbar_arrive(&ctl->tempty[buf]);
        ++use[h];
      }
    }
  }

  tc_fence_before();
  if (kPair) cluster_sync();  // both CTAs are done with each other's barriers, smem, TMEM
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

// At most 128 registers per thread: with 10 warps on the 4 SM sub-partitions (3, 3, 2, 2)
// a sub-partition holding 3 of them keeps 4096 of its 16384 registers free, room for two
// warps of a 64-register combine CTA of 8 warps -- the combine that runs beside this kernel
// must be able to reside next to it.
template <bool kSwiGLU, bool kGather, bool kTwoM>
__global__ void __maxnreg__(128)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const KParams p) {
  gemm_body<kSwiGLU, false, kGather, kTwoM>(&tmA, &tmB, &tmA, &tmB, p);
}

// Launched with a cluster of 2 CTAs (cudaLaunchAttributeClusterDimension).  The same
// register cap as the single-CTA kernel, for the combine that runs beside it.
template <bool kSwiGLU, bool kGather>
__global__ void __maxnreg__(128)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmA64,
                             const __grid_constant__ CUtensorMap tmB64, const KParams p) {
  gemm_body<kSwiGLU, true, kGather, false>(&tmA, &tmB, &tmA64, &tmB64, p);
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
// box_rows x BK columns and the matching swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int32_t cols, int32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             MOE_GEMM_L2_PROMO == 2   ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
             : MOE_GEMM_L2_PROMO == 1 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                      : CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_tma_2d_bf16(CUtensorMap* m, const void* base, int64_t rows, int32_t cols,
                      int32_t box_rows) {
  return make_map(m, base, rows, cols, box_rows);
}

bool make_tma_3d_f32(CUtensorMap* m, void* base, int32_t E, int32_t M, int32_t N) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc || N % 4 != 0) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)E};
  const cuuint64_t strides[2] = {(cuuint64_t)N * 4, (cuuint64_t)M * N * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether a GEMM kind runs on CTA pairs (MOE_GEMM_2SM bits).
bool gemm_pair(bool swiglu, bool gather) {
  const int bit = !swiglu ? 1 : (gather ? 2 : 0);
  return ((MOE_GEMM_2SM >> bit) & 1) != 0;
}

// Which single-CTA variant a GEMM kind runs: two 128-row sub-tiles per 256-row tile
// (MOE_GEMM_TWO_M bit 0: gate/up, bit 1: down) or one 128-row tile.
bool gemm_two_m(bool swiglu, bool gather) {
  if (gemm_pair(swiglu, gather)) return false;
  return ((MOE_GEMM_TWO_M >> (swiglu ? 0 : 1)) & 1) != 0;
}

bool gemm_down_lsu() { return MOE_GEMM_DOWN_LSU != 0; }

int64_t gemm_total_tiles(const int32_t* counts_host, int32_t E, int32_t out_cols, bool swiglu,
                         bool gather) {
  const int32_t bn = swiglu ? BN / 2 : BN;
  const int32_t tm = gemm_pair(swiglu, gather)    ? Geo<true>::kTileM
                     : gemm_two_m(swiglu, gather) ? Geo<false, true>::kTileM
                                                  : Geo<false>::kTileM;
  const int64_t n_tiles = (out_cols + bn - 1) / bn;
  int64_t m_tiles = 0;
  for (int32_t e = 0; e < E; ++e) m_tiles += (counts_host[e] + tm - 1) / tm;
  return m_tiles * n_tiles;
}

cudaError_t launch_grouped_gemm(const GemmArgs& a, bool swiglu, int num_sms, cudaStream_t s,
                                int* err_detail) {
  // gathered-kernel launch: rows through a map (a.gather), or A's own rows copied by the
  // gathering warps (a.gather_src set, a.gather null: the down GEMM's Act rows)
  const bool gather = a.gather != nullptr || a.gather_src != nullptr;
  const bool kPair = gemm_pair(swiglu, gather);
  const bool two_m = gemm_two_m(swiglu, gather);
  *err_detail = 0;
  // total_tiles < 0: the kernel counts them (the grid is then one CTA, or pair, per SM)
  if (a.total_tiles == 0 || a.rows <= 0) return cudaSuccess;
  if (a.total_tiles > 0x7fffffff || a.E > kMaxE || (a.total_tiles < 0 && !a.status)) {
    *err_detail = 1;
    return cudaErrorInvalidValue;
  }
  CUtensorMap mA, mB;
  const int32_t bn = swiglu ? BN / 2 : BN;
  if (gather && (a.gather_src_rows < a.rows && a.gather == nullptr)) {
    *err_detail = 1;
    return cudaErrorInvalidValue;
  }
  // (gathered A is copied by the gathering warps; its map is built but unused)
  const bool map_a_ok = gather ? make_map(&mA, a.gather_src, a.gather_src_rows, a.K, kRowsPerCta)
                               : make_map(&mA, a.A, a.rows, a.K, kRowsPerCta);
  const bool map_b_ok = make_map(&mB, a.B, (int64_t)a.E * a.b_rows, a.K,
                                 kPair ? BN / 2 : (swiglu ? BN / 2 : BN));
  // the pair's half tiles: 64-row boxes of A (each CTA's rows) and of the weights
  CUtensorMap mA64 = mA, mB64 = mB;
  const bool map_h_ok =
      !kPair || ((gather || make_map(&mA64, a.A, a.rows, a.K, kRowsPerCta / 2)) &&
                 make_map(&mB64, a.B, (int64_t)a.E * a.b_rows, a.K, BN / 4));
  if (!map_a_ok || !map_b_ok || !map_h_ok) {
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
  p.gather = a.gather;
  p.gsrc = static_cast<const uint8_t*>(a.gather_src);
  p.gsrc_stride = (int64_t)a.K * 2;
  p.gsrc_rows = a.gather_src_rows;
  p.out_rows = a.rows;
  p.K = a.K;
  const size_t smem =
      two_m ? smem_bytes<false, true>() : (kPair ? smem_bytes<true>() : smem_bytes<false>());
  cudaError_t e;
  if (kPair) {
    auto k = gather ? (swiglu ? grouped_gemm_pair_kernel<true, true>
                              : grouped_gemm_pair_kernel<false, true>)
                    : (swiglu ? grouped_gemm_pair_kernel<true, false>
                              : grouped_gemm_pair_kernel<false, false>);
    const int variant = (gather ? 2 : 0) + (swiglu ? 1 : 0);
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(gather ? gemm_threads<true>() : gemm_threads<false>(), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many CTA pairs as can be resident at once
    static int max_pairs[4][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    int& mp = max_pairs[variant][dev & 63];
    if (mp <= 0) {
      cfg.gridDim = dim3(num_sms, 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, (void*)k, &cfg) != cudaSuccess || n <= 0)
        n = num_sms / 2;
      mp = n < num_sms / 2 ? n : num_sms / 2;
    }
    const int streams = (int)(a.total_tiles >= 0 && a.total_tiles < mp ? a.total_tiles : mp);
    cfg.gridDim = dim3(2 * streams, 1, 1);
    e = cudaLaunchKernelEx(&cfg, k, mA, mB, mA64, mB64, p);
    if (e != cudaSuccess) return e;
  } else {
    auto k = two_m ? (gather ? (swiglu ? grouped_gemm_kernel<true, true, true>
                                       : grouped_gemm_kernel<false, true, true>)
                             : (swiglu ? grouped_gemm_kernel<true, false, true>
                                       : grouped_gemm_kernel<false, false, true>))
                   : (gather ? (swiglu ? grouped_gemm_kernel<true, true, false>
                                       : grouped_gemm_kernel<false, true, false>)
                             : (swiglu ? grouped_gemm_kernel<true, false, false>
                                       : grouped_gemm_kernel<false, false, false>));
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int streams =
        (int)(a.total_tiles >= 0 && a.total_tiles < num_sms ? a.total_tiles : num_sms);
    const int threads = two_m ? (gather ? gemm_threads<true, true>() : gemm_threads<false, true>())
                              : (gather ? gemm_threads<true>() : gemm_threads<false>());
    k<<<streams, threads, smem, s>>>(mA, mB, p);
  }
  return cudaGetLastError();
}

uint32_t checks_take_gemm() {
  uint32_t v = 0, zero = 0;
  if (!MOE_CHECKS) return 0;
  cudaMemcpyFromSymbol(&v, g_range_flags, sizeof v);
  cudaMemcpyToSymbol(g_range_flags, &zero, sizeof zero);
  return v;
}

}  // namespace moe
