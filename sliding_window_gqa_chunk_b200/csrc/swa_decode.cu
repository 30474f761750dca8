// swa_decode.cu - single-token decode over the rolling cache (Mistral 7B,
// section 2, Rolling Buffer Cache paragraph; token-by-token generation in the
// Pre-fill and Chunking paragraph).
//
// At position pos the new key/value go to slot pos mod W and the query attends
// over the min(pos + 1, W) cached positions (pos - W, pos].  The cache is the
// HBM-bound part: every (sequence, kv head) streams W slots x d x 2 B of keys
// and the same of values, and does ~2 x G x d FMAs per slot.  So one warp
// handles all G query heads of its kv head (the GQA group shares each load),
// and the dot products run on the tensor cores through mma.sync m16n8k16 so
// the CUDA cores only do the online softmax:
//
//   S^T[slot][head] = K[slot][:] . Q[head][:]    (M = 16 slots, N = 8 heads, K = d)
//   O^T[d][head]   += V^T[d][slot] . P^T[slot][head]  (M = 16 d, N = 8 heads, K = 16 slots)
//
// Each lane loads contiguous 16-byte pieces of K and V rows: a dot product
// over d is invariant under any permutation of d applied to both K and Q, so
// the d index is relabelled to match the mma fragment layout; the PV product
// uses a second relabelling of d (undone when O is stored) and pairs
// consecutive slots with byte permutes.  P^T goes from the S accumulator
// layout to the B-operand layout with one movmatrix.trans per 8x8 block.
// With at least one (sequence, kv head) pair per SM the pieces come straight
// from global memory (register-fed variant); with fewer pairs a producer warp
// streams each split into a shared-memory ring with bulk copies and the
// compute warps read their pieces from there (stream variant).
//
// Work split: grid (n_splits, Hkv, B); a CTA of NW warps covers one split of
// the W slots; warps take interleaved 16-slot blocks and merge their (m, l, O)
// in shared memory.  Then the CTA writes the final output (one split), or the
// splits of a (sequence, kv head) merge their partials: through distributed
// shared memory when they form a thread-block cluster (few sequences, where
// the sweep is latency-bound and a second launch would cost as much as the
// sweep), else as fp32 partials in the workspace for
// swa_decode_combine_kernel.  The CTA whose split holds slot
// pos mod W writes the new key/value there; every lane that would read that
// slot reads k_new / v_new instead, so no CTA ever reads a slot that is being
// written.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "swa_common.cuh"
#include "swa_internal.h"
#include "swa_tc.cuh"

namespace swa {

namespace {

constexpr int kBlockSlots = 16;

// Physical element offset (within a row) of lane-quad t's key piece `j`
// (K rows and Q rows use the same relabelling of d).
template <int D>
__device__ __forceinline__ int k_piece_offset(int t, int j) {
  if constexpr (D == 16) {
    return t * 4;
  } else {
    return j * 32 + t * 8;
  }
}

// Physical element offset of lane-group g's value piece `c` (PV relabelling).
template <int D>
__device__ __forceinline__ int v_piece_offset(int g, int c) {
  if constexpr (D == 16) {
    return g * 2;
  } else {
    return c * 64 + g * 8;
  }
}

template <int D>
struct Frag {
  // words of one K row held by a lane: D/4 bf16 -> D/8 words
  static constexpr int kKWords = D / 8;
  // words of one V row held by a lane: D/8 bf16 -> D/16 words
  static constexpr int kVWords = D / 16;
  static constexpr int kKSteps = D / 16;   // mma k-steps of the QK product
  static constexpr int kMTiles = D / 16;   // m-tiles of the PV product
};

// Loads the words of one row (key: kKWords, value: kVWords) into regs.
template <int D>
__device__ __forceinline__ void load_k_row(uint32_t (&w)[Frag<D>::kKWords], const __nv_bfloat16* row,
                                           int t, bool valid) {
  if constexpr (D == 16) {
    uint2 x = valid ? ldg_stream8(row + k_piece_offset<D>(t, 0)) : make_uint2(0, 0);
    w[0] = x.x;
    w[1] = x.y;
  } else {
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      uint4 x = valid ? ldg_stream(row + k_piece_offset<D>(t, j)) : make_uint4(0, 0, 0, 0);
      w[4 * j + 0] = x.x;
      w[4 * j + 1] = x.y;
      w[4 * j + 2] = x.z;
      w[4 * j + 3] = x.w;
    }
  }
}

template <int D>
__device__ __forceinline__ void load_v_row(uint32_t (&w)[Frag<D>::kVWords], const __nv_bfloat16* row,
                                           int g, bool valid) {
  if constexpr (D == 16) {
    w[0] = valid ? ldg_stream4(row + v_piece_offset<D>(g, 0)) : 0u;
  } else {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint4 x = valid ? ldg_stream(row + v_piece_offset<D>(g, c)) : make_uint4(0, 0, 0, 0);
      w[4 * c + 0] = x.x;
      w[4 * c + 1] = x.y;
      w[4 * c + 2] = x.z;
      w[4 * c + 3] = x.w;
    }
  }
}

// Stream variant: the slots come from a shared-memory ring filled by bulk
// copies.  Same fragments as load_k_row / load_v_row, read from the row at
// shared address `srow`, or from global memory `grow` for the slot the new
// key / value goes to (that slot's cache row is being rewritten).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
  return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
  return r;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(a));
  return r;
}

template <int D>
__device__ __forceinline__ void load_k_row_s(uint32_t (&w)[Frag<D>::kKWords], uint32_t srow,
                                             const __nv_bfloat16* grow, bool from_global, int t,
                                             bool valid) {
  if (!valid || from_global) {
    load_k_row<D>(w, grow, t, valid);
    return;
  }
  if constexpr (D == 16) {
    uint2 x = lds64(srow + 2 * k_piece_offset<D>(t, 0));
    w[0] = x.x;
    w[1] = x.y;
  } else {
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      uint4 x = lds128(srow + 2 * k_piece_offset<D>(t, j));
      w[4 * j + 0] = x.x;
      w[4 * j + 1] = x.y;
      w[4 * j + 2] = x.z;
      w[4 * j + 3] = x.w;
    }
  }
}

template <int D>
__device__ __forceinline__ void load_v_row_s(uint32_t (&w)[Frag<D>::kVWords], uint32_t srow,
                                             const __nv_bfloat16* grow, bool from_global, int g,
                                             bool valid) {
  if (!valid || from_global) {
    load_v_row<D>(w, grow, g, valid);
    return;
  }
  if constexpr (D == 16) {
    w[0] = lds32(srow + 2 * v_piece_offset<D>(g, 0));
  } else {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint4 x = lds128(srow + 2 * v_piece_offset<D>(g, c));
      w[4 * c + 0] = x.x;
      w[4 * c + 1] = x.y;
      w[4 * c + 2] = x.z;
      w[4 * c + 3] = x.w;
    }
  }
}

// Stream variant geometry: chunks of kChunkSlots slots (K rows and V rows,
// each one contiguous range of the cache) in a ring of kStreamStages.
constexpr int kChunkSlots = 64;
constexpr int kStreamStages = 6;

template <int D>
constexpr int stream_ring_bytes() { return kStreamStages * 2 * kChunkSlots * D * 2; }

// Compute warps of the stream variant (one more warp streams the ring).
// Warp w takes the 16-slot blocks w, w + NW, ... of its split, so it reads
// every (NW / 4)-th chunk; that stride must divide the stage count, or a warp
// could skip a fill of a stage and take a later fill's parity for an earlier
// one.  12 warps: chunks 3 apart, 2 stages per warp.
constexpr int kStreamWarps = 12;
// Groups of 9-16 query heads carry two n-tiles of accumulators per warp: 4
// compute warps (5 in all, up to 255 registers a thread, no spills).  With 12
// (at most 128 registers) the spills made a G = 16 step 25-30 % slower, with 8
// (168 registers) 2-4 %.
constexpr int kStreamWarpsWide = 4;

// Row stride (floats) of the per-warp O partials in shared memory: one float
// of padding spreads the rows that a warp's lanes store at once over the banks
// (with stride D the 4 head rows and the two halves of the d range would all
// land on the same 4 banks).
template <int D>
constexpr int merge_o_stride() { return D + 1; }
// Shared memory of the CTA merge: m, l and O of each warp, then the CTA's m, l, O.
template <int D, int NT, int NW>
constexpr int decode_merge_bytes() {
  return (int)sizeof(float) * (NW * 8 * NT * (2 + merge_o_stride<D>()) + 8 * NT * (2 + D));
}


template <typename OutT>
__device__ __forceinline__ void store_out(OutT* dst, float x);
template <>
__device__ __forceinline__ void store_out<float>(float* dst, float x) { *dst = x; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* dst, float x) {
  *dst = __float2bfloat16_rn(x);
}

}  // namespace

// NT = number of 8-head n-tiles (ceil(G / 8)); NW = compute warps.  STREAM:
// one more warp streams the CTA's slots into a shared-memory ring with bulk
// copies (every byte of the split in flight from the start), and the compute
// warps read their fragments from there.
template <int D, int NT, int NW, typename OutT, bool STREAM>
__global__ void __launch_bounds__((NW + (STREAM ? 1 : 0)) * 32)
swa_decode_kernel(const DecodeParams p) {
  using F = Frag<D>;
  extern __shared__ __align__(128) float smem[];

  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int G = p.n_q_heads / p.n_kv_heads;
  const int W = p.window;

  wait_prior_grid();
  allow_next_grid();
  const long long pos = p.pos[b];
  if (pos < 0) {
    if (threadIdx.x == 0) raise_status(p.status, SWA_ERR_DEVICE_ARG);
    return;
  }
  const int n_valid = (int)(pos + 1 < (long long)W ? pos + 1 : (long long)W);
  const int s_new = (int)(pos % W);
  const int r_begin = split * p.slots_per_split;
  const int r_stop = r_begin + p.slots_per_split;
  const int r_end = r_stop < n_valid ? r_stop : n_valid;

  const size_t head_stride = (size_t)W * D;
  const __nv_bfloat16* kc = p.k_cache + ((size_t)b * p.n_kv_heads + kvh) * head_stride;
  const __nv_bfloat16* vc = p.v_cache + ((size_t)b * p.n_kv_heads + kvh) * head_stride;
  const __nv_bfloat16* kn = p.k_new + ((size_t)b * p.n_kv_heads + kvh) * D;
  const __nv_bfloat16* vn = p.v_new + ((size_t)b * p.n_kv_heads + kvh) * D;

  // The split owning slot pos mod W stores the new key/value there.  No lane of
  // any CTA reads that slot from the cache (they read k_new / v_new).
  if (warp == 0 && s_new >= r_begin && s_new < r_stop) {
    for (int i = lane; i < D / 8; i += 32) {
      reinterpret_cast<uint4*>(p.k_cache_w + ((size_t)b * p.n_kv_heads + kvh) * head_stride +
                               (size_t)s_new * D)[i] = reinterpret_cast<const uint4*>(kn)[i];
      reinterpret_cast<uint4*>(p.v_cache_w + ((size_t)b * p.n_kv_heads + kvh) * head_stride +
                               (size_t)s_new * D)[i] = reinterpret_cast<const uint4*>(vn)[i];
    }
  }

  // ---- stream variant: ring of K / V chunks, full / empty barriers ----
  static_assert(!STREAM || ((NW * kBlockSlots) % kChunkSlots == 0 &&
                            kStreamStages % (NW * kBlockSlots / kChunkSlots) == 0),
                "a compute warp must see every fill of each ring stage it reads");
  constexpr int G8 = 8 * NT;
  constexpr int kMergeBytes = decode_merge_bytes<D, NT, NW>();
  constexpr int kOS = merge_o_stride<D>();
  constexpr int kRingBytes = STREAM ? stream_ring_bytes<D>() : 0;
  constexpr int kBarOffset = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  const uint32_t s_base = tc::smem_u32(smem);
  const uint32_t sK = s_base;
  const uint32_t sV = s_base + kStreamStages * kChunkSlots * D * 2;
  const uint32_t bar_full = s_base + kBarOffset;          // [kStreamStages]
  const uint32_t bar_empty = bar_full + 8 * kStreamStages;  // [kStreamStages]
  bool stream_ok = true;
  if constexpr (STREAM) {
    if (threadIdx.x == 0) {
      for (int i = 0; i < kStreamStages; ++i) {
        tc::mbar_init(bar_full + 8 * i, 1);
        tc::mbar_init(bar_empty + 8 * i, kChunkSlots / kBlockSlots);  // one arrival per block
      }
      tc::mbar_fence_init();
    }
    __syncthreads();
    if (warp == NW) {
      // Producer: chunk k of the split goes to stage k mod kStreamStages once
      // the blocks of chunk k - kStreamStages have been read.
      if (lane == 0) {
        const int n_slots = r_end > r_begin ? r_end - r_begin : 0;
        const int n_chunks = (n_slots + kChunkSlots - 1) / kChunkSlots;
        int k = 0;
        for (; k < n_chunks; ++k) {
          const int st = k % kStreamStages;
          if (k >= kStreamStages &&
              !tc::mbar_wait(bar_empty + 8 * st, ((k / kStreamStages) - 1) & 1, p.status)) {
            stream_ok = false;
            break;
          }
          const int x = r_begin + k * kChunkSlots;
          const int cnt = (r_end - x) < kChunkSlots ? (r_end - x) : kChunkSlots;
          const uint32_t bytes = (uint32_t)cnt * D * 2;
          tc::mbar_arrive_expect_tx(bar_full + 8 * st, 2 * bytes);
          tc::bulk_load(sK + st * kChunkSlots * D * 2, kc + (size_t)x * D, bytes, bar_full + 8 * st);
          tc::bulk_load(sV + st * kChunkSlots * D * 2, vc + (size_t)x * D, bytes, bar_full + 8 * st);
        }
        // every copy issued here has landed before the ring is reused
        for (int j = k > kStreamStages ? k - kStreamStages : 0; j < k; ++j)
          tc::mbar_wait(bar_full + 8 * (j % kStreamStages), (j / kStreamStages) & 1, p.status);
      }
    }
  }

  // Q as the B operand of S^T = K Q^T: lane (g, t) holds head 8*nt + g.
  uint32_t qf[NT][F::kKWords];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hl = nt * 8 + g;
    const bool hv = hl < G;
    const __nv_bfloat16* qrow = p.q + ((size_t)b * p.n_q_heads + (size_t)kvh * G + (hv ? hl : 0)) * D;
    load_k_row<D>(qf[nt], qrow, t, hv);
  }

  float o[NT][F::kMTiles][4];
  float m_run[NT][2];
  float l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int mt = 0; mt < F::kMTiles; ++mt) {
      o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    }
    m_run[nt][0] = m_run[nt][1] = -CUDART_INF_F;
    l_run[nt][0] = l_run[nt][1] = 0.f;
  }
  const float sl2 = p.scale_log2;

  const int loop_end = (STREAM && warp >= NW) ? r_begin : r_end;  // the producer warp computes nothing
  for (int blk = r_begin + warp * kBlockSlots; blk < loop_end; blk += NW * kBlockSlots) {
    // ---- loads: K rows blk+g, blk+8+g; V rows blk+2t, +1, +8, +9 ----
    uint32_t kw0[F::kKWords], kw1[F::kKWords];
    uint32_t vw[4][F::kVWords];
    if constexpr (STREAM) {
      const int k = (blk - r_begin) / kChunkSlots;
      const int st = k % kStreamStages;
      stream_ok = __all_sync(0xffffffffu,
                             tc::mbar_wait(bar_full + 8 * st, (k / kStreamStages) & 1, p.status));
      if (!stream_ok) break;
      const int in0 = blk - r_begin - k * kChunkSlots;  // first row of the block within the chunk
      const uint32_t ks = sK + st * kChunkSlots * D * 2 + in0 * D * 2;
      const uint32_t vs = sV + st * kChunkSlots * D * 2 + in0 * D * 2;
      const int r0 = blk + g, r1 = blk + 8 + g;
      load_k_row_s<D>(kw0, ks + g * D * 2, kn, r0 == s_new, t, r0 < r_end);
      load_k_row_s<D>(kw1, ks + (8 + g) * D * 2, kn, r1 == s_new, t, r1 < r_end);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ri = 2 * t + (i & 1) + (i >> 1) * 8;
        const int r = blk + ri;
        load_v_row_s<D>(vw[i], vs + ri * D * 2, vn, r == s_new, g, r < r_end);
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_empty + 8 * st);  // this block's rows are in registers
    } else {
      const int r0 = blk + g, r1 = blk + 8 + g;
      load_k_row<D>(kw0, r0 == s_new ? kn : kc + (size_t)r0 * D, t, r0 < r_end);
      load_k_row<D>(kw1, r1 == s_new ? kn : kc + (size_t)r1 * D, t, r1 < r_end);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = blk + 2 * t + (i & 1) + (i >> 1) * 8;
        load_v_row<D>(vw[i], r == s_new ? vn : vc + (size_t)r * D, g, r < r_end);
      }
    }
    const bool ok0 = blk + g < r_end;
    const bool ok1 = blk + 8 + g < r_end;

    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < F::kKSteps; ++ks) {
        // k-step ks uses words 2*ks and 2*ks+1 of each row's piece list
        mma_16816(s, kw0[2 * ks], kw1[2 * ks], kw0[2 * ks + 1], kw1[2 * ks + 1],
                  qf[nt][2 * ks], qf[nt][2 * ks + 1]);
      }
      // s[0]: (slot g, head 2t)   s[1]: (slot g, head 2t+1)
      // s[2]: (slot g+8, head 2t) s[3]: (slot g+8, head 2t+1)
      s[0] = ok0 ? s[0] * sl2 : -CUDART_INF_F;
      s[1] = ok0 ? s[1] * sl2 : -CUDART_INF_F;
      s[2] = ok1 ? s[2] * sl2 : -CUDART_INF_F;
      s[3] = ok1 ? s[3] * sl2 : -CUDART_INF_F;
      float mx0 = fmaxf(s[0], s[2]);
      float mx1 = fmaxf(s[1], s[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[nt][0], mx0);
      const float mn1 = fmaxf(m_run[nt][1], mx1);
      const float a0 = fast_exp2(m_run[nt][0] - mn0);
      const float a1 = fast_exp2(m_run[nt][1] - mn1);
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
      const float p0 = fast_exp2(s[0] - mn0);
      const float p1 = fast_exp2(s[1] - mn1);
      const float p2 = fast_exp2(s[2] - mn0);
      const float p3 = fast_exp2(s[3] - mn1);
      l_run[nt][0] = l_run[nt][0] * a0 + p0 + p2;
      l_run[nt][1] = l_run[nt][1] * a1 + p1 + p3;
#pragma unroll
      for (int mt = 0; mt < F::kMTiles; ++mt) {
        o[nt][mt][0] *= a0;
        o[nt][mt][1] *= a1;
        o[nt][mt][2] *= a0;
        o[nt][mt][3] *= a1;
      }
      pb[nt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
      pb[nt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
    }

    // ---- O^T += V^T P^T ----
#pragma unroll
    for (int mt = 0; mt < F::kMTiles; ++mt) {
      const int c = (D == 16) ? 0 : mt / 4;
      const int qq = (D == 16) ? 0 : mt % 4;
      const uint32_t w0 = vw[0][4 * c + qq], w1 = vw[1][4 * c + qq];
      const uint32_t w2 = vw[2][4 * c + qq], w3 = vw[3][4 * c + qq];
      const uint32_t a0 = prmt(w0, w1, 0x5410);
      const uint32_t a1 = prmt(w0, w1, 0x7632);
      const uint32_t a2 = prmt(w2, w3, 0x5410);
      const uint32_t a3 = prmt(w2, w3, 0x7632);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(o[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
  }

  // ---- merge the NW warps of the CTA ----
  // smem: m[NW][G8], l[NW][G8], O[NW][G8][kOS] with G8 = 8*NT, then the CTA's
  // partial m[G8], l[G8], O[G8][D] (cluster merge); in the stream variant this
  // reuses the ring, once every warp is done with it.
  if constexpr (STREAM) {
    if (!stream_ok && lane == 0) raise_status(p.status, SWA_ERR_TIMEOUT);
    __syncthreads();
  }
  float* sm_m = smem;
  float* sm_l = sm_m + NW * G8;
  float* sm_o = sm_l + NW * G8;
  float* cta_m = sm_o + (size_t)NW * G8 * kOS;
  float* cta_l = cta_m + G8;
  float* cta_o = cta_l + G8;
#pragma unroll
  for (int nt = 0; nt < NT && warp < NW; ++nt) {
    float l0 = l_run[nt][0], l1 = l_run[nt][1];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const int h0 = nt * 8 + 2 * t;
    if (g == 0) {
      sm_m[warp * G8 + h0] = m_run[nt][0];
      sm_m[warp * G8 + h0 + 1] = m_run[nt][1];
      sm_l[warp * G8 + h0] = l0;
      sm_l[warp * G8 + h0 + 1] = l1;
    }
#pragma unroll
    for (int mt = 0; mt < F::kMTiles; ++mt) {
      // logical rows (mt, g) and (mt, g+8) -> physical d
      int d0;
      if constexpr (D == 16) {
        d0 = 2 * g;
      } else {
        d0 = (mt / 4) * 64 + g * 8 + (mt % 4) * 2;
      }
      float* oh0 = sm_o + ((size_t)warp * G8 + h0) * kOS;
      float* oh1 = oh0 + kOS;
      oh0[d0] = o[nt][mt][0];
      oh1[d0] = o[nt][mt][1];
      oh0[d0 + 1] = o[nt][mt][2];
      oh1[d0 + 1] = o[nt][mt][3];
    }
  }
  __syncthreads();

  const int hq0 = kvh * G;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int h = idx / D;
    const int dd = idx - h * D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w * G8 + h]);
    float L = 0.f, O = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float sc = fast_exp2(sm_m[w * G8 + h] - M);
        L += sc * sm_l[w * G8 + h];
        O += sc * sm_o[((size_t)w * G8 + h) * kOS + dd];
      }
    }
    const size_t bh = (size_t)b * p.n_q_heads + hq0 + h;
    if (p.n_splits == 1) {
      store_out<OutT>(reinterpret_cast<OutT*>(p.out) + bh * D + dd, O / L);
    } else if (p.cluster) {
      cta_o[h * D + dd] = O;
      if (dd == 0) {
        cta_m[h] = M;
        cta_l[h] = L;
      }
    } else {
      p.ws_o[(bh * p.n_splits + split) * D + dd] = O;
      if (dd == 0) {
        p.ws_ml[(bh * p.n_splits + split) * 2 + 0] = M;
        p.ws_ml[(bh * p.n_splits + split) * 2 + 1] = L;
      }
    }
  }

  if (p.cluster) {
    // The n_splits CTAs of this (sequence, kv head) are one cluster: each
    // merges a share of the G x d outputs from every CTA's partial, read
    // through distributed shared memory.  Every CTA of the cluster reaches
    // both barriers (no CTA of a cluster returns early: they share pos).
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    const int rank = (int)cl.block_rank();
    const int R = p.n_splits;
    // Rank r merges outputs [r * per, (r + 1) * per) of the G x d outputs, so
    // every CTA takes an equal share; each thread fetches all R partials of
    // its output with independent remote loads before combining them.
    const int per = (G * D + R - 1) / R;
    for (int idx = rank * per + threadIdx.x; idx < (rank + 1) * per && idx < G * D; idx += blockDim.x) {
      const int h = idx / D;
      const int dd = idx - h * D;
      float m_r[kDecodeMaxClusterSplits], l_r[kDecodeMaxClusterSplits], o_r[kDecodeMaxClusterSplits];
#pragma unroll
      for (int r = 0; r < kDecodeMaxClusterSplits; ++r) {
        if (r < R) {
          m_r[r] = cl.map_shared_rank(cta_m, r)[h];
          l_r[r] = cl.map_shared_rank(cta_l, r)[h];
          o_r[r] = cl.map_shared_rank(cta_o, r)[h * D + dd];
        } else {
          m_r[r] = -CUDART_INF_F;
          l_r[r] = o_r[r] = 0.f;
        }
      }
      float M = -CUDART_INF_F;
#pragma unroll
      for (int r = 0; r < kDecodeMaxClusterSplits; ++r) M = fmaxf(M, m_r[r]);
      float L = 0.f, O = 0.f;
      if (M != -CUDART_INF_F) {
#pragma unroll
        for (int r = 0; r < kDecodeMaxClusterSplits; ++r) {
          const float sc = (m_r[r] == -CUDART_INF_F) ? 0.f : fast_exp2(m_r[r] - M);
          L += sc * l_r[r];
          O += sc * o_r[r];
        }
      }
      const size_t bh = (size_t)b * p.n_q_heads + hq0 + h;
      store_out<OutT>(reinterpret_cast<OutT*>(p.out) + bh * D + dd, O / L);
    }
    cl.sync();  // keep this CTA's partial alive until every peer has read it
  }
}

// Merge of the per-split partials: grid (B * Hq), one thread per d.
template <int D, typename OutT>
__global__ void __launch_bounds__(D < 32 ? 32 : D)
swa_decode_combine_kernel(const DecodeParams p) {
  wait_prior_grid();
  allow_next_grid();
  const size_t bh = blockIdx.x;
  const int dd = threadIdx.x;
  if (dd >= D) return;
  const int S = p.n_splits;
  const float* ml = p.ws_ml + bh * S * 2;
  float M = -CUDART_INF_F;
  for (int s = 0; s < S; ++s) M = fmaxf(M, ml[2 * s]);
  float L = 0.f, O = 0.f;
  const float* op = p.ws_o + bh * S * D + dd;
  for (int s = 0; s < S; ++s) {
    const float m = ml[2 * s];
    if (m == -CUDART_INF_F) continue;
    const float sc = fast_exp2(m - M);
    L += sc * ml[2 * s + 1];
    O += sc * op[(size_t)s * D];
  }
  store_out<OutT>(reinterpret_cast<OutT*>(p.out) + bh * D + dd, O / L);
}

namespace {

constexpr int kMaxDevices = 64;

template <int D, int NT, int NW, typename OutT, bool STREAM>
cudaError_t launch_decode_t(const DecodeParams& p, cudaStream_t stream) {
  constexpr size_t merge = (size_t)decode_merge_bytes<D, NT, NW>();
  constexpr size_t ring = STREAM ? (size_t)stream_ring_bytes<D>() : 0;
  constexpr size_t smem = (ring > merge ? ring : merge) + (STREAM ? 16 * kStreamStages : 0);
  auto kern = swa_decode_kernel<D, NT, NW, OutT, STREAM>;
  if (smem > 48 * 1024) {
    // raised once per device (the attribute persists for the process)
    static bool set[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!set[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      set[dev] = true;
    }
  }
  dim3 grid(p.n_splits, p.n_kv_heads, p.batch);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.n_splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3((NW + (STREAM ? 1 : 0)) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = p.cluster ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess || p.n_splits == 1 || p.cluster) return e;
  cudaLaunchConfig_t ccfg = {};
  ccfg.gridDim = dim3((unsigned)((size_t)p.batch * p.n_q_heads));
  ccfg.blockDim = dim3(D < 32 ? 32 : D);
  ccfg.stream = stream;
  ccfg.attrs = attr;
  ccfg.numAttrs = 1;
  return cudaLaunchKernelEx(&ccfg, swa_decode_combine_kernel<D, OutT>, p);
}

template <int D, typename OutT>
cudaError_t launch_decode_d(const DecodeParams& p, cudaStream_t stream) {
  const int G = p.n_q_heads / p.n_kv_heads;
  if (p.stream) {
    if (G <= 8) return launch_decode_t<D, 1, kStreamWarps, OutT, true>(p, stream);
    return launch_decode_t<D, 2, kStreamWarpsWide, OutT, true>(p, stream);
  }
  if (G <= 8) return launch_decode_t<D, 1, 4, OutT, false>(p, stream);
  return launch_decode_t<D, 2, 4, OutT, false>(p, stream);
}

template <typename OutT>
cudaError_t launch_decode_o(const DecodeParams& p, cudaStream_t stream) {
  switch (p.head_dim) {
    case 16: return launch_decode_d<16, OutT>(p, stream);
    case 64: return launch_decode_d<64, OutT>(p, stream);
    case 128: return launch_decode_d<128, OutT>(p, stream);
  }
  return cudaErrorInvalidValue;
}

template <int D>
int resident_clusters_d(int cs) {
  auto kern = swa_decode_kernel<D, 1, kStreamWarps, __nv_bfloat16, true>;
  constexpr size_t merge = (size_t)decode_merge_bytes<D, 1, kStreamWarps>();
  constexpr size_t ring = (size_t)stream_ring_bytes<D>();
  constexpr size_t smem = (ring > merge ? ring : merge) + 16 * kStreamStages;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return -1;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cs);
  cfg.blockDim = dim3((kStreamWarps + 1) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return -1;
  return n;
}

}  // namespace

int decode_resident_clusters(int head_dim, int cs) {
  if (cs < 1 || cs > kDecodeMaxClusterSplits) return -1;
  const int di = head_dim == 16 ? 0 : head_dim == 64 ? 1 : head_dim == 128 ? 2 : -1;
  int dev = 0;
  if (di < 0 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();  // no device: leave no error behind for the next call
    return -1;
  }
  // answers per device, head dimension and cluster size (value + 1; 0 = not asked yet)
  static int cache[kMaxDevices][3][kDecodeMaxClusterSplits + 1] = {};
  int& c = cache[dev][di][cs];
  if (c == 0) {
    int n = -1;
    switch (head_dim) {
      case 16: n = resident_clusters_d<16>(cs); break;
      case 64: n = resident_clusters_d<64>(cs); break;
      default: n = resident_clusters_d<128>(cs); break;
    }
    if (n < 0) {
      cudaGetLastError();
      return -1;
    }
    c = n + 1;
  }
  return c - 1;
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream) {
  if (p.out_f32) return launch_decode_o<float>(p, stream);
  return launch_decode_o<__nv_bfloat16>(p, stream);
}

}  // namespace swa
