// swa_prefill.cu - attention of one prefill chunk over the rolling cache and the
// chunk itself (Mistral 7B, section 2, Pre-fill and Chunking paragraph and
// Figure 3), on the 5th-generation tensor cores of sm_100a.
//
// A unit of work is one 128-row query tile of one or two query heads that
// share a kv head (GQA: both heads reuse every K/V tile the CTA loads) of one
// sequence.  With a workspace the grid is one CTA per SM and each CTA takes
// units, heaviest first, from a counter in the workspace; the units of the
// last wave are cut into pieces of their key range whose partial softmax
// results are merged by log-sum-exp.  Without one, the grid has one CTA per
// unit.  Warp roles:
//   warps 0-3  softmax for head slot 0 (TMEM lanes 0-127 = the 128 query rows)
//   warps 4-7  softmax for head slot 1
//   warp  8    TMA producer: Q of each unit, then K tiles into an NK-stage ring
//   warp  9    TMEM allocator and MMA issuer (one elected lane issues tcgen05.mma)
//   warp 10    TMA producer: V tiles into an NV-stage ring
//   warp 11    work fetcher: takes units (or pieces of units) and publishes
//              them to the other roles through a two-entry ring
// The kernel is compiled for 168 registers per thread (12 warps); the third
// warpgroup gives registers back (setmaxnreg) so that each softmax thread can
// hold its whole 128-column row of S without spilling.
// Per key tile j and head slot i:
//   S_i = Q_i K_j^T       tcgen05.mma, A = Q (smem), B = K (smem), D = S_i (TMEM, fp32)
//   softmax warps read S_i row by row (one thread per query row), mask, update
//   the running max / sum (rescaling O_i only when the max grows by more than
//   2^8), and write P_i = exp2(...) as bf16 back over S_i in TMEM
//   O_i += P_i V_j        tcgen05.mma, A = P (TMEM), B = V (smem, d-contiguous)
// Tensor memory: S_0 | S_1 | O_0 | O_1  (128 + 128 + d + d columns of 512).
// The epilogue divides O_i by the row sum; whole 128-row tiles of bf16 output
// at d = 128 leave through a shared-memory staging tile and TMA stores, other
// rows are stored from registers.
//
// Key tiles: the keys of a chunk are the cache slots holding positions
// [max(0, s + t_lo - W + 1), s) and the chunk rows [0, t_hi].  The cache
// positions form one cyclic range of slots, so they are covered by 128-slot
// tiles starting at slot-tile index first and wrapping past the last one: the
// modular index p mod W goes straight into the TMA row coordinate.  Tiles that
// no query row of the CTA can see are never loaded; inside the loaded tiles
// each row masks the keys outside its own window [i - W + 1, i] and, in the
// chunk, the keys after it (causal).
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "swa_common.cuh"
#include "swa_exp2.cuh"
#include "swa_internal.h"
#include "swa_tc.cuh"

namespace swa {

namespace {

// Progress words for debugging hangs: compiled in only with -DSWA_TRACE, where
// p.trace points at host-mapped memory the host can read while a kernel runs.
#ifdef SWA_TRACE
#define SWA_TRACE_AT(slot, value)                                                             \
  do {                                                                                        \
    if (p.trace != nullptr) {                                                                 \
      const int cta_ = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;       \
      *reinterpret_cast<volatile int*>(p.trace + cta_ * 8 + (slot)) = (value);                \
      __threadfence_system();                                                                 \
    }                                                                                         \
  } while (0)
#else
#define SWA_TRACE_AT(slot, value) \
  do {                            \
  } while (0)
#endif

// Bits [lo, hi) of the 32 keys that start at key w0, as a mask.
__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int w0) {
  int l = lo - w0, h = hi - w0;
  l = l < 0 ? 0 : (l > 32 ? 32 : l);
  h = h < 0 ? 0 : (h > 32 ? 32 : h);
  if (h <= l) return 0u;
  const uint32_t hm = h >= 32 ? 0xffffffffu : ((1u << h) - 1u);
  const uint32_t lm = l >= 32 ? 0xffffffffu : ((1u << l) - 1u);
  return hm & ~lm;
}

constexpr int kRows = 128;          // query rows per tile = TMEM lanes
constexpr int kKeys = 128;          // keys per tile
constexpr int kThreads = 384;       // 12 warps = 3 warpgroups
// Register split: launched at kLaunchRegs per thread, the two softmax
// warpgroups grow to kSoftmaxRegs and the producer/MMA warpgroup shrinks to
// kOtherRegs.  2 * kSoftmaxRegs + kOtherRegs must equal 3 * kLaunchRegs (the
// block's register pool), or setmaxnreg.inc would wait forever; the host
// refuses to launch if ptxas did not allocate exactly kLaunchRegs.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
constexpr int kOtherRegs = 88;
static_assert(2 * kSoftmaxRegs + kOtherRegs == 3 * kLaunchRegs, "register split must fill the pool");
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr int kFetchWarp = 11;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
// A row's sum of p over one tile above which the optimistic exponentials are
// redone against the tile's own max (2^32: far below fp32 overflow, so no p of
// the optimistic pass can have overflowed unnoticed).
constexpr float kOptimisticSumLimit = 4294967296.0f;
constexpr uint32_t kTmemCols = 512;
// Workspace layout: two scheduler counters; one merge counter per split unit
// and softmax warp (at most one split unit per persistent CTA); then one fp32
// partial result slot per key-range piece (at most one per persistent CTA):
// per head, O^T [d][128 rows] followed by the running max [128] and sum [128].
constexpr int kMaxPersistentCtas = 256;
// A unit of the split tail is cut into pieces only if it has at least this
// many key tiles; lighter units go whole to their first piece.
constexpr int kMinSplitTiles = 8;
constexpr size_t kWsMergeOffset = 256;
constexpr size_t kWsPartialOffset = 16384;
static_assert(kWsMergeOffset + kMaxPersistentCtas * 8 * sizeof(int) <= kWsPartialOffset, "workspace layout");
// Which of every 8 consecutive (even, odd) column pairs take the FMA-pipe
// exp2 (swa_exp2.cuh) instead of the SFU: bit w set means pair w mod 8.  The
// SFU's exp2 has a quarter of the FMA pipe's lane rate, so moving a fraction
// of the pairs shortens the softmax pass.  Both paths give exactly 0 for a
// masked key (-inf).
#ifndef SWA_EXP2_FMA_PAIRS
#define SWA_EXP2_FMA_PAIRS 0x00
#endif

// K / V ring depths for head_dim 128 (2 Q tiles + K + V must fit in 227 KB).
#ifndef SWA_K_STAGES_D128
#define SWA_K_STAGES_D128 2
#endif
#ifndef SWA_V_STAGES_D128
#define SWA_V_STAGES_D128 2
#endif

template <int D>
struct Cfg {
  static constexpr int kSwzBytes = (D * 2 >= 128) ? 128 : D * 2;  // swizzle span = bytes per box row
  static constexpr int kBoxD = kSwzBytes / 2;                      // d-elements per TMA box row
  static constexpr int kColBlocks = (D * 2) / kSwzBytes;          // boxes per 128-row tile
  static constexpr int kBlockBytes = kRows * kSwzBytes;           // one box
  static constexpr int kTileBytes = kRows * D * 2;                // one 128 x d bf16 tile
  // K and V rings are separate: a K tile is released as soon as the S
  // products of both heads have consumed it, a V tile after the PV products.
  static constexpr int kKStages = (D == 128) ? SWA_K_STAGES_D128 : 4;
  static constexpr int kVStages = (D == 128) ? SWA_V_STAGES_D128 : 4;
  static constexpr uint32_t kLayout = (kSwzBytes == 128) ? tc::kLayoutSW128 : tc::kLayoutSW32;
  static constexpr int kSBO = 8 * kSwzBytes;                       // stride of 8-row groups
  static constexpr int kKStepsPerBlock = kSwzBytes / 32;           // 16-element k-steps per box row
  // d = 128: one 128 x d bf16 tile of shared memory stages a head's output
  // for a TMA store (the two head slots take turns)
  static constexpr int kStageBytes = (D == 128) ? kTileBytes : 0;
  static constexpr int kSmemTiles = (2 + kKStages + kVStages) * kTileBytes + kStageBytes;
  static constexpr int kSmemBytes = kSmemTiles + 512 + 1024;       // barriers + alignment slack
  static_assert(kColBlocks * kSwzBytes == D * 2, "head_dim must fill whole swizzle rows");
};

// The key tiles of one CTA, in issue order: cache tiles (cyclic over slot
// tiles), then chunk tiles 0..qt.  Every role evaluates the same plan.
struct TilePlan {
  int n_cache;
  int first_cache;
  int n_wtiles;
  int n_chunk;
  __device__ __forceinline__ int total() const { return n_cache + n_chunk; }
  __device__ __forceinline__ void at(int j, bool& is_cache, int& base) const {
    if (j < n_cache) {
      int ti = first_cache + j;
      if (ti >= n_wtiles) ti -= n_wtiles;
      is_cache = true;
      base = ti * kKeys;
    } else {
      is_cache = false;
      base = (j - n_cache) * kKeys;
    }
  }
};

__device__ __forceinline__ TilePlan make_plan(long long s, int t_lo, int qt, int W) {
  TilePlan pl;
  pl.n_wtiles = (W + kKeys - 1) / kKeys;
  pl.n_chunk = qt + 1;
  long long c_lo = s + t_lo - W + 1;
  if (c_lo < 0) c_lo = 0;
  const long long n_c = s - c_lo;  // cache positions some row of the tile can see
  if (n_c <= 0) {
    pl.n_cache = 0;
    pl.first_cache = 0;
    return pl;
  }
  // Positions are below 2^32 (start_pos is an int32 and t < W), so the
  // slot arithmetic runs in 32-bit unsigned (a 64-bit remainder is a long
  // subroutine that would cost the producer warps registers).
  const int a = (int)((uint32_t)c_lo % (uint32_t)W);
  const int last = (int)((uint32_t)(c_lo + n_c - 1) % (uint32_t)W);
  const int ft = a / kKeys, lt = last / kKeys;
  if (a + n_c <= W) {
    pl.first_cache = ft;
    pl.n_cache = lt - ft + 1;
  } else if (lt < ft) {
    pl.first_cache = ft;
    pl.n_cache = (pl.n_wtiles - ft) + lt + 1;
  } else {
    pl.first_cache = 0;
    pl.n_cache = pl.n_wtiles;
  }
  return pl;
}

template <typename OutT>
__device__ __forceinline__ void store16(OutT* dst, const float (&v)[16], float scale, bool v8);

// 32 bytes in one instruction (sm_100 256-bit store); dst must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* dst, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

template <>
__device__ __forceinline__ void store16<float>(float* dst, const float (&v)[16], float scale, bool v8) {
  if (v8) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(v[8 * i + e] * scale);
      st_global_v8(dst + 8 * i, w);
    }
    return;
  }
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d4[i] = make_float4(v[4 * i] * scale, v[4 * i + 1] * scale, v[4 * i + 2] * scale,
                        v[4 * i + 3] * scale);
}

template <>
__device__ __forceinline__ void store16<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[16],
                                                       float scale, bool v8) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(v[2 * e] * scale, v[2 * e + 1] * scale);
  if (v8) {
    st_global_v8(dst, w);
    return;
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
}


// One work item: a piece of one unit (a 128-row query tile of one sequence and
// one head pair).  Units are numbered heaviest first: query tile index
// descending (in a chunk that starts its prompt tile qt sees qt + 1 key
// tiles), then sequence, then head pair.  Items [0, n_whole) are whole units;
// the last units are split into n_pieces pieces that take consecutive parts of
// the unit's key tiles, and their partial softmax results are merged by the
// piece that finishes last.
struct Item {
  int b, qt, kvh, h_first, t_lo;
  long long s;        // start position of the chunk
  int n;              // tokens of the sequence in this chunk
  bool rows;          // the unit has query rows to compute
  bool bad_args;      // start_pos / n_tokens out of range for this sequence
  int piece, np;      // piece index and piece count (np == 1: whole unit)
  int merge_idx;      // split unit index (merge counters)
  int slot;           // partial result slot of this piece
  int j0, n_tiles;    // the piece's tiles: plan tiles [j0, j0 + n_tiles)
  TilePlan plan;
};

__device__ __forceinline__ Item decode_item(const PrefillParams& p, int item) {
  Item it;
  int u;
  if (item < p.n_whole) {
    u = item;
    it.piece = 0;
    it.np = 1;
    it.merge_idx = 0;
    it.slot = 0;
  } else {
    const int k = item - p.n_whole;
    u = p.n_whole + k / p.n_pieces;
    it.piece = k % p.n_pieces;
    it.np = p.n_pieces;
    it.merge_idx = k / p.n_pieces;
    it.slot = k;
  }
  const int hpc = p.heads_per_cta;
  const int nhp = p.n_q_heads / hpc;
  const int per_qt = p.batch * nhp;
  it.qt = p.n_q_tiles - 1 - u / per_qt;
  const int r = u - (u / per_qt) * per_qt;
  it.b = r / nhp;
  const int hp = r - it.b * nhp;
  const int G = p.n_q_heads / p.n_kv_heads;
  const int pairs = G / hpc;
  it.kvh = hp / pairs;
  it.h_first = it.kvh * G + (hp - it.kvh * pairs) * hpc;
  it.t_lo = it.qt * kRows;
  it.s = p.start_pos[it.b];
  it.n = p.n_tokens[it.b];
  it.bad_args = it.s < 0 || it.n < 0 || it.n > p.max_tokens;
  it.rows = !it.bad_args && it.t_lo < it.n;
  it.j0 = 0;
  it.n_tiles = 0;
  it.plan.n_cache = it.plan.first_cache = it.plan.n_chunk = 0;
  it.plan.n_wtiles = 1;
  if (it.rows) {
    it.plan = make_plan(it.s, it.t_lo, it.qt, p.window);
    const int w = it.plan.total();
    if (it.np > 1 && w < kMinSplitTiles) {
      // Too few key tiles to be worth a merge (a causal first chunk's
      // lightest tiles): piece 0 takes the whole unit, the others nothing.
      it.rows = it.piece == 0;
      it.np = 1;
      if (!it.rows) return it;
    }
    it.j0 = (int)((long long)it.piece * w / it.np);
    it.n_tiles = (int)((long long)(it.piece + 1) * w / it.np) - it.j0;
  }
  return it;
}

// Partial result slot of one piece and head: O^T [D][128 rows], then the
// running max [128] and sum [128] (log2 domain, as the softmax keeps them).
template <int D>
__device__ __forceinline__ float* partial_slot(const PrefillParams& p, int slot, int head) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(p.workspace) + kWsPartialOffset) +
         ((size_t)slot * p.heads_per_cta + head) * (size_t)(kRows * (D + 2));
}

__device__ __forceinline__ float ld_cg(const float* a) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(a));
  return v;
}

// An item as the fetcher warp publishes it in shared memory: the fields every
// role needs, so that no other role repeats the decoding (its divisions and
// global loads would sit on the critical path of each item and cost
// registers in the producer warpgroup).
constexpr int kRecInts = 20;
enum RecField {
  kRecEnd = 0, kRecB, kRecKvh, kRecHFirst, kRecTLo, kRecS, kRecN, kRecPiece, kRecNp, kRecMerge,
  kRecSlot, kRecJ0, kRecNTiles, kRecNCache, kRecFirstCache, kRecNWTiles, kRecNChunk
};

__device__ __forceinline__ void rec_store(volatile int* r, const Item& I, bool end) {
  r[kRecEnd] = end ? 1 : 0;
  if (end) return;
  r[kRecB] = I.b;
  r[kRecKvh] = I.kvh;
  r[kRecHFirst] = I.h_first;
  r[kRecTLo] = I.t_lo;
  r[kRecS] = (int)I.s;
  r[kRecN] = I.n;
  r[kRecPiece] = I.piece;
  r[kRecNp] = I.np;
  r[kRecMerge] = I.merge_idx;
  r[kRecSlot] = I.slot;
  r[kRecJ0] = I.j0;
  r[kRecNTiles] = I.n_tiles;
  r[kRecNCache] = I.plan.n_cache;
  r[kRecFirstCache] = I.plan.first_cache;
  r[kRecNWTiles] = I.plan.n_wtiles;
  r[kRecNChunk] = I.plan.n_chunk;
}

__device__ __forceinline__ Item rec_load(const volatile int* r) {
  Item I;
  I.b = r[kRecB];
  I.kvh = r[kRecKvh];
  I.h_first = r[kRecHFirst];
  I.t_lo = r[kRecTLo];
  I.qt = I.t_lo / kRows;
  I.s = r[kRecS];
  I.n = r[kRecN];
  I.rows = true;
  I.bad_args = false;
  I.piece = r[kRecPiece];
  I.np = r[kRecNp];
  I.merge_idx = r[kRecMerge];
  I.slot = r[kRecSlot];
  I.j0 = r[kRecJ0];
  I.n_tiles = r[kRecNTiles];
  I.plan.n_cache = r[kRecNCache];
  I.plan.first_cache = r[kRecFirstCache];
  I.plan.n_wtiles = r[kRecNWTiles];
  I.plan.n_chunk = r[kRecNChunk];
  return I;
}

}  // namespace

template <int D, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
swa_prefill_kernel(const PrefillParams p, const __grid_constant__ PrefillMaps maps) {
  using C = Cfg<D>;
  constexpr int NK = C::kKStages;
  constexpr int NV = C::kVStages;
  extern __shared__ uint8_t smem_raw[];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int hpc = p.heads_per_cta;
  const int W = p.window;
  int* const ws_ctr = static_cast<int*>(p.workspace);  // [0] next item, [1] CTAs done

  // ---- shared memory carve-up (1024-byte aligned for the 128B swizzle) ----
  const uint32_t raw_addr = tc::smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_addr);
  const uint32_t sQ = base;                                   // 2 tiles
  const uint32_t sK = base + 2 * C::kTileBytes;               // NK tiles
  const uint32_t sV = sK + NK * C::kTileBytes;                // NV tiles
  const uint32_t sStage = sV + NV * C::kTileBytes;            // output staging tile (d = 128)
  const uint32_t sBar = base + C::kSmemTiles;
  // barrier addresses (8 bytes each)
  const uint32_t bar_q_full = sBar;
  const uint32_t bar_q_empty = sBar + 8;
  const uint32_t bar_k_full = sBar + 16;               // [NK]
  const uint32_t bar_k_empty = bar_k_full + 8 * NK;    // [NK]
  const uint32_t bar_v_full = bar_k_empty + 8 * NK;    // [NV]
  const uint32_t bar_v_empty = bar_v_full + 8 * NV;    // [NV]
  const uint32_t bar_s_full = bar_v_empty + 8 * NV;    // [2]
  const uint32_t bar_p_full = bar_s_full + 16;         // [2]
  const uint32_t bar_o_full = bar_p_full + 16;         // [2]
  const uint32_t bar_item_full = bar_o_full + 16;      // [2]
  const uint32_t bar_item_empty = bar_item_full + 16;  // [2]
  const uint32_t bar_done = bar_item_empty + 16;
  const uint32_t bar_fetch = bar_done + 8;             // K producer done issuing an item
  const uint32_t bar_stage_free = bar_fetch + 8;       // the staging tile has been read by its TMA store
  const uint32_t bar_stage_full = bar_stage_free + 8;  // [2] a head slot's rows are in the staging tile
  static_assert(16 + 16 * NK + 16 * NV + 5 * 16 + 40 <= 320, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kSmemTiles + 320);
  volatile int* item_rec = reinterpret_cast<volatile int*>(base_ptr + C::kSmemTiles + 336);  // [2][kRecInts]
  static_assert(336 + 2 * kRecInts * 4 <= 512, "item records must fit the control area");
  // Consumers of the item queue: the K and V producers, the MMA warp and
  // every softmax warp (one arrival each).
  const int n_item_consumers = 3 + 4 * hpc;

  if (threadIdx.x == 0) {
    tc::mbar_init(bar_q_full, 1);
    tc::mbar_init(bar_q_empty, 1);
    for (int i = 0; i < NK; ++i) {
      tc::mbar_init(bar_k_full + 8 * i, 1);
      tc::mbar_init(bar_k_empty + 8 * i, 1);
    }
    for (int i = 0; i < NV; ++i) {
      tc::mbar_init(bar_v_full + 8 * i, 1);
      tc::mbar_init(bar_v_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(bar_s_full + 8 * i, 1);
      tc::mbar_init(bar_p_full + 8 * i, kRows / 32);  // one arrival per softmax warp
      tc::mbar_init(bar_o_full + 8 * i, 1);
      tc::mbar_init(bar_item_full + 8 * i, 1);
      tc::mbar_init(bar_item_empty + 8 * i, n_item_consumers);
    }
    tc::mbar_init(bar_done, 1);
    tc::mbar_init(bar_fetch, 1);
    tc::mbar_init(bar_stage_free, 1);
    tc::mbar_init(bar_stage_full, kRows / 32);
    tc::mbar_init(bar_stage_full + 8, kRows / 32);
    tc::mbar_fence_init();
  }
  if (threadIdx.x == 0) SWA_TRACE_AT(0, 1);
  if (warp == kMmaWarp) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
    if (lane == 0) SWA_TRACE_AT(0, 2);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) SWA_TRACE_AT(0, 3);
  // Launched with programmatic stream serialization: the set-up above (no
  // global memory) may overlap the previous kernel; nothing below reads or
  // writes global memory before that kernel has completed.
  wait_prior_grid();
  allow_next_grid();

  // Item queue: the fetcher warp takes items (the CTA's own index first, then
  // from the shared counter when the grid is persistent), skips units with no
  // query rows, and publishes each remaining item as a record in a two-entry
  // ring; every other role reads the same sequence.  A record with the end
  // flag closes it.  Consumers read the fields they need before they release
  // the entry.
  auto wait_item = [&](int it, bool& ok) -> const volatile int* {
    const int slot = it & 1;
    ok = tc::mbar_wait(bar_item_full + 8 * slot, (it >> 1) & 1, p.status);
    return item_rec + slot * kRecInts;
  };

  // setmaxnreg is per warpgroup and must dominate the code it budgets, so the
  // role dispatch happens inside the two register branches.
  if (warp >= 8) {
  tc::regs_decrease<kOtherRegs>();
  if (warp == kFetchWarp) {
    // ================================ item fetcher ================================
    if (lane == 0) {
      bool ok = true;
      int pub = 0;  // records published
      for (int fetch = 0; ok; ++fetch) {
        int item = p.n_items;
        // Take the next unit only once the K producer has issued the last
        // tile of the previous one (a few tiles before the CTA finishes it),
        // so that units go to CTAs close to the moment they can start them:
        // greedy longest-first over the SMs, not a round-robin two units deep.
        if (pub > 0 && fetch > 0) {
          ok = tc::mbar_wait(bar_fetch, (pub - 1) & 1, p.status);
          if (!ok) break;
        }
        if (fetch == 0) {
          item = blockIdx.x;
        } else if (p.persistent) {
          const int got = atomicAdd(ws_ctr, 1);
          // A counter below zero means the workspace was not zero-filled:
          // stop instead of walking an unbounded item range.
          if (got < 0) raise_status(p.status, SWA_ERR_DEVICE_ARG);
          else item = (int)gridDim.x + got;
        }
        if (item > p.n_items) item = p.n_items;
        const bool end = item >= p.n_items;
        Item I;
        if (!end) {
          I = decode_item(p, item);
          if (I.bad_args && I.qt == 0 && I.piece == 0 && I.h_first == 0)
            raise_status(p.status, SWA_ERR_DEVICE_ARG);
          if (!I.rows) continue;  // no query rows: nothing for the other roles
        }
        const int slot = pub & 1;
        if (pub >= 2) ok = tc::mbar_wait(bar_item_empty + 8 * slot, ((pub >> 1) - 1) & 1, p.status);
        if (!ok) break;
        rec_store(item_rec + slot * kRecInts, I, end);
        tc::mbar_arrive(bar_item_full + 8 * slot);
        ++pub;
        if (end) break;
      }
    }
  } else if (warp == kProducerWarp) {
    // ======================== TMA producer: Q, then K tiles ========================
    if (lane == 0) {
      tc::prefetch_map(&maps.q);
      tc::prefetch_map(&maps.k);
      tc::prefetch_map(&maps.kc);
      int kt = 0;   // K tiles issued (ring position)
      int qi = 0;   // Q tiles issued (items with tiles)
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const volatile int* rec = wait_item(it, ok);
        if (!ok) break;
        const bool end = rec[kRecEnd] != 0;
        Item I;
        if (!end) I = rec_load(rec);
        tc::mbar_arrive(bar_item_empty + 8 * (it & 1));
        if (end) break;
        if (I.n_tiles == 0) {
          tc::mbar_arrive(bar_fetch);
          continue;
        }
        SWA_TRACE_AT(1, 1000 + it);
        if (qi > 0) ok = tc::mbar_wait(bar_q_empty, (qi - 1) & 1, p.status);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(bar_q_full, hpc * C::kTileBytes);
        for (int i = 0; i < hpc; ++i)
          for (int cb = 0; cb < C::kColBlocks; ++cb)
            tc::tma_load_4d(sQ + i * C::kTileBytes + cb * C::kBlockBytes, &maps.q, cb * C::kBoxD,
                            I.h_first + i, I.t_lo, I.b, bar_q_full);
        ++qi;
        for (int j = 0; j < I.n_tiles; ++j, ++kt) {
          bool is_cache;
          int kbase;
          I.plan.at(I.j0 + j, is_cache, kbase);
          const int sk = kt % NK;
          if (kt >= NK) ok = tc::mbar_wait(bar_k_empty + 8 * sk, ((kt / NK) - 1) & 1, p.status);
          if (!ok) break;
          const uint32_t kdst = sK + sk * C::kTileBytes;
          tc::mbar_arrive_expect_tx(bar_k_full + 8 * sk, C::kTileBytes);
#ifdef SWA_TILE_COUNTERS
          if (p.trace != nullptr) atomicAdd(p.trace, 1);  // checked build: key tiles loaded
#endif
          for (int cb = 0; cb < C::kColBlocks; ++cb) {
            if (is_cache)
              tc::tma_load_3d(kdst + cb * C::kBlockBytes, &maps.kc, cb * C::kBoxD, kbase,
                              I.b * p.n_kv_heads + I.kvh, bar_k_full + 8 * sk);
            else
              tc::tma_load_4d(kdst + cb * C::kBlockBytes, &maps.k, cb * C::kBoxD, I.kvh, kbase, I.b,
                              bar_k_full + 8 * sk);
          }
        }
        if (ok) tc::mbar_arrive(bar_fetch);  // the fetcher may take the next unit now
      }
      // Before leaving, make sure no copy issued here is still in flight: the
      // last Q load and the last use of every K stage.
      SWA_TRACE_AT(1, 5000);
      if (qi > 0) tc::mbar_wait(bar_q_full, (qi - 1) & 1, p.status);
      for (int j = kt > NK ? kt - NK : 0; j < kt; ++j)
        tc::mbar_wait(bar_k_full + 8 * (j % NK), (j / NK) & 1, p.status);
      SWA_TRACE_AT(1, 9999);
    }
  } else if (warp == kVProducerWarp) {
    // ========================= TMA producer: V tiles =========================
    // A separate issuer, so that a K load never waits behind a V stage that is
    // still being read (the V ring turns over one iteration later than K's).
    if (lane == 0) {
      tc::prefetch_map(&maps.v);
      tc::prefetch_map(&maps.vc);
      int vt = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const volatile int* rec = wait_item(it, ok);
        if (!ok) break;
        const bool end = rec[kRecEnd] != 0;
        Item I;
        if (!end) I = rec_load(rec);
        tc::mbar_arrive(bar_item_empty + 8 * (it & 1));
        if (end) break;
        for (int j = 0; j < I.n_tiles; ++j, ++vt) {
          bool is_cache;
          int kbase;
          I.plan.at(I.j0 + j, is_cache, kbase);
          const int sv = vt % NV;
          if (vt >= NV) ok = tc::mbar_wait(bar_v_empty + 8 * sv, ((vt / NV) - 1) & 1, p.status);
          if (!ok) break;
          const uint32_t vdst = sV + sv * C::kTileBytes;
          tc::mbar_arrive_expect_tx(bar_v_full + 8 * sv, C::kTileBytes);
          for (int cb = 0; cb < C::kColBlocks; ++cb) {
            if (is_cache)
              tc::tma_load_3d(vdst + cb * C::kBlockBytes, &maps.vc, cb * C::kBoxD, kbase,
                              I.b * p.n_kv_heads + I.kvh, bar_v_full + 8 * sv);
            else
              tc::tma_load_4d(vdst + cb * C::kBlockBytes, &maps.v, cb * C::kBoxD, I.kvh, kbase, I.b,
                              bar_v_full + 8 * sv);
          }
        }
      }
      for (int j = vt > NV ? vt - NV : 0; j < vt; ++j)
        tc::mbar_wait(bar_v_full + 8 * (j % NV), (j / NV) & 1, p.status);
    }
  } else if (warp == kMmaWarp) {
    // ============================ MMA issuer ============================
    // The whole warp runs this loop converged (warp-uniform waits); one
    // elected lane issues each tcgen05.mma / commit.
    {
      constexpr uint32_t idesc_s = tc::make_idesc_bf16(kRows, kKeys, false, false);
      constexpr uint32_t idesc_pv = tc::make_idesc_bf16(kRows, D, false, true);
      // Shared-memory descriptors are built once; a k-step or a stage only
      // moves the start address, i.e. adds (bytes >> 4) to the low field
      // (shared addresses stay below 2^18, so the 14-bit field never carries).
      const uint64_t q_desc = tc::make_sdesc(sQ, 16, C::kSBO, C::kLayout);
      const uint64_t k_desc = tc::make_sdesc(sK, 16, C::kSBO, C::kLayout);
      const uint64_t v_desc = tc::make_sdesc(sV, C::kBlockBytes, C::kSBO, C::kLayout);
      auto issue_s = [&](int i, int st) {
        const uint32_t d_tmem = tmem + i * kKeys;
        const uint64_t qd = q_desc + (uint64_t)((i * C::kTileBytes) >> 4);
        const uint64_t kd = k_desc + (uint64_t)((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int cb = ks / C::kKStepsPerBlock;
          const int kin = ks % C::kKStepsPerBlock;
          const uint64_t off = (uint64_t)((cb * C::kBlockBytes + kin * 32) >> 4);
          tc::mma_ss_elect(d_tmem, qd + off, kd + off, idesc_s, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int st, bool accumulate) {
        const uint32_t d_tmem = tmem + 2 * kKeys + i * D;
        const uint32_t a_tmem = tmem + i * kKeys;
        const uint64_t vd = v_desc + (uint64_t)((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < kKeys / 16; ++ks) {
          const uint64_t off = (uint64_t)((ks * 16 * C::kSwzBytes) >> 4);
          tc::mma_ts_elect(d_tmem, a_tmem + ks * 8, vd + off, idesc_pv, (accumulate || ks > 0) ? 1u : 0u);
        }
      };

      SWA_TRACE_AT(2, 10);
      int kt = 0;   // K tiles consumed
      int vt = 0;   // V tiles consumed
      int g0 = 0;   // S tiles before the current item (S / P barrier phases)
      int qi = 0;   // items with tiles
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const volatile int* rec;
        {
          bool got;
          rec = wait_item(it, got);
          ok = __all_sync(0xffffffffu, got);
        }
        if (!ok) break;
        const bool end = rec[kRecEnd] != 0;
        const int n_tiles = end ? 0 : rec[kRecNTiles];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_item_empty + 8 * (it & 1));
        if (end) break;
        if (n_tiles == 0) continue;
        ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_q_full, qi & 1, p.status));
        if (!ok) break;
        ++qi;
        tc::tc_fence_after();
        // Per tile j: for each head slot i, O_i += P_i(j-1) V(j-1) (needs the
        // softmax of tile j-1), then S_i(j) = Q_i K(j)^T.  A tcgen05.commit
        // tracks every MMA issued before it, so the V stage is released right
        // after the last PV that reads it, the K stage right after the last S,
        // and the Q tiles after the item's last S.
        for (int j = 0; j <= n_tiles && ok; ++j) {
          const bool has_s = j < n_tiles;
          const int sk = kt % NK;
          if (has_s) {
            SWA_TRACE_AT(2, 1000 + j);
            ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_k_full + 8 * sk, (kt / NK) & 1, p.status));
            if (!ok) break;
          }
          const int svp = vt % NV;
          // V(j - 1) is checked while the softmax of tile j - 1 still runs, so
          // that the P V products follow the P-ready arrivals directly.
          if (j > 0)
            ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_v_full + 8 * svp, (vt / NV) & 1, p.status));
          for (int i = 0; i < hpc && ok; ++i) {
            if (j > 0) {
              ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_p_full + 8 * i, (g0 + j - 1) & 1, p.status));
              if (!ok) break;
              tc::tc_fence_after();
              issue_pv(i, svp, j - 1 > 0);
              if (i == hpc - 1) tc::tc_commit_elect(bar_v_empty + 8 * svp);
              if (!has_s) tc::tc_commit_elect(bar_o_full + 8 * i);
            }
            if (has_s) {
              tc::tc_fence_after();
              SWA_TRACE_AT(2, 3000 + j * 2 + i);
              issue_s(i, sk);
              tc::tc_commit_elect(bar_s_full + 8 * i);
            }
          }
          if (!ok) break;
          if (has_s) {
            tc::tc_commit_elect(bar_k_empty + 8 * sk);
            ++kt;
            if (j == n_tiles - 1) tc::tc_commit_elect(bar_q_empty);
          }
          if (j > 0) ++vt;
        }
        g0 += n_tiles;
      }
      // All MMAs must have finished before the TMEM is released.
      SWA_TRACE_AT(2, 8000);
      tc::tc_commit_elect(bar_done);
      tc::mbar_wait(bar_done, 0, p.status);
      SWA_TRACE_AT(2, 9999);
    }
  }
  } else {
  tc::regs_increase<kSoftmaxRegs>();
  if (warp / 4 < hpc) {
    // ============================ softmax / epilogue ============================
    const int i = warp / 4;                   // head slot
    const int row = (warp % 4) * 32 + lane;   // query row within the tile = TMEM lane
    const uint32_t lane_addr = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + i * kKeys;
    const uint32_t tO = tmem + lane_addr + 2 * kKeys + i * D;
    const float sl2 = p.scale_log2;
    int g0 = 0;   // S tiles before the current item
    int oi = 0;   // items with tiles (O barrier phase)
    int n_staged = 0;  // items whose output went through the staging tile
    bool stage_pending = false;  // this thread's TMA store may still be reading the staging tile
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const volatile int* rec;
      {
        bool got;
        rec = wait_item(it, got);
        ok = __all_sync(0xffffffffu, got);
      }
      if (!ok) break;
      const bool end = rec[kRecEnd] != 0;
      Item I;
      if (!end) I = rec_load(rec);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_item_empty + 8 * (it & 1));
      if (end) break;
      const int n_tiles = I.n_tiles;
      const int t = I.t_lo + row;               // chunk row
      if (stage_pending) {
        // the other head slot may use the staging tile once this store has read it
        tc::bulk_wait_read_all();
        tc::mbar_arrive(bar_stage_free);
        stage_pending = false;
      }
      const long long s = I.s;
      const long long pos_i = s + t;            // absolute query position
      // this row's visible cache slots: the cyclic range [a_i, a_i + len_i)
      long long lo_i = pos_i - W + 1;
      if (lo_i < 0) lo_i = 0;
      const int len_i = (int)(s - lo_i);          // <= W - 1; <= 0 means none
      const int a_i = (int)((uint32_t)lo_i % (uint32_t)W);

      float m_run = -CUDART_INF_F;
      float l_run = 0.f;
      for (int j = 0; j < n_tiles; ++j) {
        if (row == 0) SWA_TRACE_AT(3 + i, 1000 + j);
        // tcgen05.ld / st / wait are warp-collective (.sync.aligned): every
        // decision that guards them must be the same on all 32 lanes.
        ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_s_full + 8 * i, (g0 + j) & 1, p.status));
        if (!ok) break;
        tc::tc_fence_after();
        float sv[kKeys];
        {
          float* chunk = sv;
#pragma unroll
          for (int c = 0; c < kKeys / 32; ++c)
            tc::tmem_ld32(tS + c * 32, *reinterpret_cast<float(*)[32]>(chunk + c * 32));
        }
        tc::tc_wait_ld();
#pragma unroll
        for (int c = 0; c < kKeys / 16; ++c) tc::reg_fence16(sv + c * 16);

        bool is_cache;
        int kbase;
        I.plan.at(I.j0 + j, is_cache, kbase);
        // Visible keys of this row in this tile: [v_lo0, v_hi0) U [v_lo1, v_hi1).
        // A cache tile: slot kbase + k is visible iff it is < W and
        // (kbase + k - a_i) mod W < len_i, i.e. k < len_i - d0, or
        // W - d0 <= k < W - d0 + len_i.  A chunk tile: key kbase + k <= t.
        bool masked = false;  // this row has invisible keys in this tile
        int v_lo0 = 0, v_hi0 = kKeys, v_lo1 = 0, v_hi1 = 0;
        if (is_cache) {
          int d0 = kbase - a_i;
          if (d0 < 0) d0 += W;
          masked = !((kbase + kKeys <= W) && (len_i > 0) && (d0 + kKeys <= len_i));
          const int r_end = W - kbase;
          v_hi0 = min(len_i - d0, r_end);
          v_lo1 = W - d0;
          v_hi1 = min(W - d0 + len_i, r_end);
        } else {
          masked = kbase + kKeys - 1 > t;
          v_hi0 = t - kbase + 1;
        }
        if (masked) {
          // as four 32-bit visibility words, then one select per score
          uint32_t vm[kKeys / 32];
#pragma unroll
          for (int w = 0; w < kKeys / 32; ++w)
            vm[w] = range_bits(v_lo0, v_hi0, 32 * w) | range_bits(v_lo1, v_hi1, 32 * w);
#pragma unroll
          for (int k = 0; k < kKeys; ++k)
            sv[k] = ((vm[k >> 5] >> (k & 31)) & 1u) ? sv[k] : -CUDART_INF_F;
        }
#ifdef SWA_TILE_COUNTERS
        {  // checked build: (warp, tile) pairs with / without a masked key
          const bool wm = __any_sync(0xffffffffu, masked);
          if (lane == 0 && p.trace != nullptr) atomicAdd(p.trace + (wm ? 1 : 2), 1);
        }
#endif

        // P = exp2(scale * log2(e) * s - base) for the whole tile, written over
        // the first 64 columns of S_i; returns this thread's sum of the fp32 p.
        auto exp_pass = [&](float base_neg) -> float {
          const uint64_t sl2x2 = f2_pack(sl2, sl2);
          const uint64_t nbx2 = f2_pack(base_neg, base_neg);
          uint64_t lsum[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < kKeys / 32; ++c) {
            uint32_t pw[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
              const float s0 = sv[c * 32 + 2 * w], s1 = sv[c * 32 + 2 * w + 1];
              const uint64_t x = f2_fma(f2_pack(s0, s1), sl2x2, nbx2);
              float p0, p1;
              f2_unpack(x, p0, p1);
              if ((SWA_EXP2_FMA_PAIRS >> (w % 8)) & 1) {
                exp2_fma_pipe(p0, p1);
              } else {
                p0 = fast_exp2(p0);
                p1 = fast_exp2(p1);
              }
              lsum[w & 1] = f2_add(lsum[w & 1], f2_pack(p0, p1));
              pw[w] = pack_bf16x2(p0, p1);
            }
            tc::tmem_st16(tS + c * 16, pw);  // P (bf16 pairs) over the first 64 columns of S_i
          }
          float a0, a1, b0, b1;
          f2_unpack(lsum[0], a0, a1);
          f2_unpack(lsum[1], b0, b1);
          return (a0 + a1) + (b0 + b1);
        };

        // Optimistic pass: exponentiate against the running max right away and
        // look at the row's sum of p afterwards.  The running max may be stale
        // (it moves only when a row's max grows by more than 2^8), so p can
        // exceed 1; bf16 and fp32 keep their relative precision at any such
        // scale.  A sum above 2^32, which any p above 2^32 (or an overflowed
        // one) produces, sends the tile to the exact pass, as does a row's
        // first visible tile.  The decisions are warp-uniform because the TMEM
        // accesses they guard are warp-collective.
        float part = 0.f;
        bool exact = __any_sync(0xffffffffu, m_run == -CUDART_INF_F);
        if (!exact) {
          part = exp_pass(-m_run);
          exact = __any_sync(0xffffffffu, !(part <= kOptimisticSumLimit));
        }
        if (exact) {
          // row maximum: 8 independent 3-input max chains, then a short tree
          float mx8[8];
#pragma unroll
          for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(sv[a], sv[8 + a]);
#pragma unroll
          for (int k = 16; k < kKeys; k += 16) {
#pragma unroll
            for (int a = 0; a < 8; ++a) mx8[a] = fmax3(mx8[a], sv[k + a], sv[k + 8 + a]);
          }
          const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                 fmaxf(mx8[6], mx8[7]));
          const float m_new = fmaxf(m_run, mx * sl2);
          // Rescale only when this row's max grew by more than 2^8; otherwise keep
          // the stale max (p <= 2^8 stays exact enough in bf16 and fp32).
          const bool grow = m_new > m_run + kRescaleThreshold;
          float alpha = 1.f;
          if (grow) {
            alpha = fast_exp2(m_run - m_new);  // 0 while nothing was visible yet
            l_run *= alpha;
            m_run = m_new;
          }
          if (j > 0 && __any_sync(0xffffffffu, grow)) {
            // O_i holds this item's previous tiles (its last PV finished before
            // S_i(j) did).  The whole warp takes this branch; rows that keep
            // their max multiply by 1.
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
              float ov[16];
              tc::tmem_ld16(tO + c * 16, ov);
              tc::tc_wait_ld();
              tc::reg_fence16(ov);
              uint32_t ow[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) ow[e] = __float_as_uint(ov[e] * alpha);
              tc::tmem_st16(tO + c * 16, ow);
            }
          }
          part = exp_pass((m_run == -CUDART_INF_F) ? 0.f : -m_run);
        }
        l_run += part;
        tc::tc_wait_st();
        tc::tc_fence_before();
        __syncwarp();
#ifdef SWA_TEST_FAULTS
        // Checked build for the timeout test: with the fault switch on, softmax
        // warp 0 withholds its P-ready arrival on the last tile of its first
        // item, so the MMA warp's bounded wait runs out.  No copy is withheld.
        const bool withhold = p.trace != nullptr && *p.trace == 1 && warp == 0 && it == 0 &&
                              j == n_tiles - 1;
        if (lane == 0 && !withhold) tc::mbar_arrive(bar_p_full + 8 * i);
#else
        if (lane == 0) tc::mbar_arrive(bar_p_full + 8 * i);
#endif
        if (row == 0) SWA_TRACE_AT(3 + i, 2000 + j);
      }
      if (!ok) break;
      g0 += n_tiles;

      // ---------------------------------- epilogue ----------------------------------
      if (row == 0) SWA_TRACE_AT(3 + i, 7000);
      const bool have_o = n_tiles > 0;
      if (have_o) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_o_full + 8 * i, oi & 1, p.status));
        ++oi;
        if (!ok) break;
        tc::tc_fence_after();
      }
      OutT* dst = reinterpret_cast<OutT*>(p.out) +
                  (((size_t)I.b * p.max_tokens + t) * p.n_q_heads + (I.h_first + i)) * D;
      if (I.np == 1) {
        const float inv_l = 1.f / l_run;
        // the whole row of O in one batch of loads and one wait
        float ov[D];
#pragma unroll
        for (int c = 0; c < D / 16; ++c)
          tc::tmem_ld16(tO + c * 16, *reinterpret_cast<float(*)[16]>(ov + c * 16));
        tc::tc_wait_ld();
#pragma unroll
        for (int c = 0; c < D / 16; ++c) tc::reg_fence16(ov + c * 16);
        if (C::kStageBytes > 0 && p.out_tma && I.t_lo + kRows <= I.n) {
          // A whole tile of bf16 output: the head's rows go to the staging
          // tile in the TMA box layout (128-byte swizzle: 16-byte chunk c of
          // row r at (c ^ (r mod 8)) * 16), then one thread stores each column
          // block with a TMA store.  The head slots take turns on the tile.
          const int use = n_staged * hpc + i;
          ++n_staged;
          if (use > 0) {
            ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_stage_free, (use - 1) & 1, p.status));
            if (!ok) break;
          }
#pragma unroll
          for (int cb = 0; cb < C::kColBlocks; ++cb) {
#pragma unroll
            for (int c = 0; c < C::kSwzBytes / 16; ++c) {
              const float* v8 = ov + cb * C::kBoxD + c * 8;
              tc::st_shared_v4(sStage + cb * C::kBlockBytes + row * C::kSwzBytes + ((c ^ (row & 7)) << 4),
                               pack_bf16x2(v8[0] * inv_l, v8[1] * inv_l), pack_bf16x2(v8[2] * inv_l, v8[3] * inv_l),
                               pack_bf16x2(v8[4] * inv_l, v8[5] * inv_l), pack_bf16x2(v8[6] * inv_l, v8[7] * inv_l));
            }
          }
          // Each warp's writes reach the async proxy, then the warp counts
          // itself; the head slot's first warp waits (bounded) for all four
          // and issues the stores.
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(bar_stage_full + 8 * i);
          if ((warp & 3) == 0) {
            ok = __all_sync(0xffffffffu, tc::mbar_wait(bar_stage_full + 8 * i, (n_staged - 1) & 1, p.status));
            if (!ok) break;
            if (lane == 0) {
#pragma unroll
              for (int cb = 0; cb < C::kColBlocks; ++cb)
                tc::tma_store_4d(&maps.out, cb * C::kBoxD, I.h_first + i, I.t_lo, I.b,
                                 sStage + cb * C::kBlockBytes);
              tc::bulk_commit_group();
              stage_pending = true;  // released below, once the next item is under way
            }
            __syncwarp();
          }
          continue;
        }
        if (t < I.n) {
#pragma unroll
          for (int c = 0; c < D / 16; ++c)
            store16<OutT>(dst + c * 16, *reinterpret_cast<const float(*)[16]>(ov + c * 16), inv_l,
                          p.out_v8 != 0);
        }
        continue;
      }
      // A piece of a split unit: publish this warp's 32 rows of (O, max, sum),
      // then count the pieces that have done so; the warp that completes the
      // count merges every piece's rows (its own straight from TMEM) and
      // writes the output.  Each warp merges its own rows, so warps never wait
      // for one another.
      const float m_own = have_o ? m_run : -CUDART_INF_F;
      const float l_own = have_o ? l_run : 0.f;
      {
        float* part = partial_slot<D>(p, I.slot, i);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          float ov[16];
          if (have_o) {
            tc::tmem_ld16(tO + c * 16, ov);
            tc::tc_wait_ld();
            tc::reg_fence16(ov);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = 0.f;
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) part[(c * 16 + e) * kRows + row] = ov[e];
        }
        part[D * kRows + row] = m_own;
        part[D * kRows + kRows + row] = l_own;
      }
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        int* ctr = reinterpret_cast<int*>(static_cast<uint8_t*>(p.workspace) + kWsMergeOffset) +
                   I.merge_idx * 8 + (warp & 7);
        const int old = atomicAdd(ctr, 1);
        last = old == I.np - 1;
        if (last) atomicExch(ctr, 0);  // leave the counter zero for the next call
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (!last) continue;
      __threadfence();
      const int slot0 = I.slot - I.piece;
      float M = m_own;
      for (int q = 0; q < I.np; ++q)
        if (q != I.piece) M = fmaxf(M, ld_cg(partial_slot<D>(p, slot0 + q, i) + D * kRows + row));
      float a_own = (m_own == -CUDART_INF_F) ? 0.f : fast_exp2(m_own - M);
      float L = a_own * l_own;
      float a_q[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a_q[q] = 0.f;
        if (q < I.np && q != I.piece) {
          const float* pq = partial_slot<D>(p, slot0 + q, i);
          const float mq = ld_cg(pq + D * kRows + row);
          a_q[q] = (mq == -CUDART_INF_F) ? 0.f : fast_exp2(mq - M);
          L += a_q[q] * ld_cg(pq + D * kRows + kRows + row);
        }
      }
      const float inv_l = 1.f / L;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        float ov[16];
        if (have_o) {
          tc::tmem_ld16(tO + c * 16, ov);
          tc::tc_wait_ld();
          tc::reg_fence16(ov);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) ov[e] = have_o ? ov[e] * a_own : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q < I.np && q != I.piece && a_q[q] != 0.f) {
            const float* pq = partial_slot<D>(p, slot0 + q, i) + (c * 16) * kRows + row;
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] += a_q[q] * ld_cg(pq + e * kRows);
          }
        }
        if (t < I.n) store16<OutT>(dst + c * 16, ov, inv_l, p.out_v8 != 0);
      }
    }
    // every TMA store of the output has completed before the CTA leaves
    if ((warp & 3) == 0 && lane == 0) tc::bulk_wait_all();
    if (stage_pending) tc::mbar_arrive(bar_stage_free);
    if (row == 0) SWA_TRACE_AT(3 + i, ok ? 8000 : 7500);
  }
  }

  tc::tc_fence_before();
  if (threadIdx.x == 0) SWA_TRACE_AT(5, 1);
  __syncthreads();
  if (threadIdx.x == 0) SWA_TRACE_AT(5, 2);
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
    if (lane == 0) SWA_TRACE_AT(5, 3);
  }
  if (threadIdx.x == 0 && p.persistent) {
    // The last CTA to finish resets the scheduler counters for the next call
    // (every CTA has made its last fetch before it gets here).
    __threadfence();
    if (atomicAdd(ws_ctr + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(ws_ctr, 0);
      atomicExch(ws_ctr + 1, 0);
    }
  }
}

namespace {

// Per device: SM count, and which kernel instantiations had their dynamic
// shared memory limit raised (set once per device, not per launch).
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {};

template <int D, typename OutT>
cudaError_t launch_prefill_t(const PrefillParams& p, const PrefillMaps& maps, int grid, int device,
                             cudaStream_t stream) {
  using C = Cfg<D>;
  auto kern = swa_prefill_kernel<D, OutT>;
  // The setmaxnreg split assumes the launch register count; never launch with another.
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes attr;
    cudaError_t ea = cudaFuncGetAttributes(&attr, kern);
    if (ea != cudaSuccess) return ea;
    regs = attr.numRegs;
  }
  if (regs != kLaunchRegs) return cudaErrorInvalidKernelImage;
  static bool smem_set[kMaxDevices] = {};
  if (!smem_set[device]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    smem_set[device] = true;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, maps);
}

template <typename OutT>
cudaError_t launch_prefill_o(const PrefillParams& p, const PrefillMaps& maps, int grid, int device,
                             cudaStream_t stream) {
  switch (p.head_dim) {
    case 16: return launch_prefill_t<16, OutT>(p, maps, grid, device, stream);
    case 64: return launch_prefill_t<64, OutT>(p, maps, grid, device, stream);
    case 128: return launch_prefill_t<128, OutT>(p, maps, grid, device, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t prefill_workspace_bytes(int hpc, int d) {
  return kWsPartialOffset + (size_t)kMaxPersistentCtas * hpc * kRows * (d + 2) * sizeof(float);
}

void prefill_map_geometry(int head_dim, int* box_elems, int* swizzle_bytes) {
  const int swz = (head_dim * 2 >= 128) ? 128 : head_dim * 2;
  *swizzle_bytes = swz;
  *box_elems = swz / 2;
}

PrefillSchedule prefill_schedule(long long n_units, int n_wtiles, int n_sms, bool have_workspace) {
  PrefillSchedule sc;
  sc.n_whole = n_units;
  sc.n_pieces = 1;
  sc.n_items = n_units;
  sc.persistent = 0;
  sc.grid = n_units;
  if (!have_workspace || n_units < 1) return sc;
  long long ctas = n_sms < kMaxPersistentCtas ? n_sms : kMaxPersistentCtas;
  if (ctas < 1) ctas = 1;
  // Units are taken heaviest first, so the last wave over the SMs is the one
  // that can leave SMs idle (with fewer units than SMs, the only wave).  Its
  // units (the last `tail` in the order) are cut into pieces of their key
  // range so that the round fills the SMs: at most ctas pieces in all, at most
  // 4 per unit, about 4 or more key tiles each for a unit that sees a whole
  // window (n_wtiles + 1 tiles).
  const long long tail = n_units % ctas;
  long long pieces = 1;
  if (tail > 0) {
    pieces = ctas / tail;
    if (pieces > 4) pieces = 4;
    const long long by_size = (n_wtiles + 1) / 4;
    if (pieces > by_size) pieces = by_size;
    if (pieces < 1) pieces = 1;
  }
  if (pieces > 1) {
    sc.n_whole = n_units - tail;
    sc.n_pieces = (int)pieces;
  }
  sc.n_items = sc.n_whole + (n_units - sc.n_whole) * sc.n_pieces;
  sc.persistent = 1;
  sc.grid = ctas < sc.n_items ? ctas : sc.n_items;
  return sc;
}

cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& maps, int grid, cudaStream_t stream) {
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  if (p.out_f32) return launch_prefill_o<float>(p, maps, grid, device, stream);
  return launch_prefill_o<__nv_bfloat16>(p, maps, grid, device, stream);
}

int device_sm_count(int device) {
  if (device < 0 || device >= kMaxDevices) return 0;
  if (g_sm_count[device] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return 0;
    g_sm_count[device] = n;
  }
  return g_sm_count[device];
}

}  // namespace swa
