// swa_internal.h - launch parameter blocks shared between the C-ABI layer
// (swa_api.cu) and the kernel files.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace swa {

struct AppendParams {
  __nv_bfloat16* k_cache;       // [B][Hkv][W][d]
  __nv_bfloat16* v_cache;
  const __nv_bfloat16* k;       // [B][max_tokens][Hkv][d]
  const __nv_bfloat16* v;
  const int32_t* start_pos;     // device [B]
  const int32_t* n_tokens;      // device [B]
  int* status;                  // device status word
  int batch, n_kv_heads, head_dim, window, max_tokens;
};

struct DecodeParams {
  void* out;                    // [B][Hq][d] bf16 or f32
  const __nv_bfloat16* q;       // [B][Hq][d]
  const __nv_bfloat16* k_new;   // [B][Hkv][d]
  const __nv_bfloat16* v_new;
  const __nv_bfloat16* k_cache; // [B][Hkv][W][d] (read path)
  const __nv_bfloat16* v_cache;
  __nv_bfloat16* k_cache_w;     // same buffers (write of slot pos mod W)
  __nv_bfloat16* v_cache_w;
  const int32_t* pos;           // device [B]
  float* ws_o;                  // [B][Hq][n_splits][d] partial O (n_splits > 1)
  float* ws_ml;                 // [B][Hq][n_splits][2] partial (max, sum), log2 domain
  int* status;
  int batch, n_q_heads, n_kv_heads, head_dim, window;
  int n_splits, slots_per_split;
  int warps;                    // warps per CTA
  int cluster;                  // 1: the n_splits CTAs of a (sequence, kv head) form a
                                // thread-block cluster and merge through distributed
                                // shared memory (no workspace, no combine kernel)
  int stream;                   // 1: a producer warp streams the slots into shared
                                // memory with bulk copies (few (sequence, kv head) pairs)
  float scale_log2;             // scale * log2(e)
  int out_f32;
};

// Largest thread-block cluster of decode split CTAs (the portable cluster size).
constexpr int kDecodeMaxClusterSplits = 8;

// Split of the W slots of one (sequence, kv head) across CTAs; depends only
// on the shape so that the workspace size is a function of the dims.
struct DecodeSplit {
  int n_splits;
  int slots_per_split;
  int warps;
  int cluster;
  int stream;
  int ws_splits;   // splits the workspace is sized for (fp32 partials per split)
};
DecodeSplit decode_split(int batch, int n_q_heads, int n_kv_heads, int window, int head_dim);

// Thread-block clusters of `cs` stream-variant decode CTAs (head dimension
// head_dim) that the current device holds at once, or -1 when it cannot be
// asked (no device).
int decode_resident_clusters(int head_dim, int cs);

struct PrefillParams {
  void* out;                    // [B][max_tokens][Hq][d] bf16 or f32
  const int32_t* start_pos;     // device [B]
  const int32_t* n_tokens;      // device [B]
  int* status;
  int batch, n_q_heads, n_kv_heads, head_dim, window, max_tokens;
  int heads_per_cta;            // 1 or 2 query heads of one kv group per CTA
  int n_q_tiles;                // ceil(max_tokens / 128)
  int n_whole;                  // work items that are whole units (query tile x head pair x sequence)
  int n_pieces;                 // pieces per split unit (units n_whole.. are split)
  int n_items;                  // total work items
  int persistent;               // 1: CTAs take items from the workspace counter
  float scale_log2;
  int out_f32;
  int out_v8;                   // 1: out is 32-byte aligned (the epilogue stores 32 bytes per instruction)
  int out_tma;                  // 1: whole output tiles go out through shared memory and a TMA
                                // store (bf16 output, d = 128; maps.out is encoded)
  void* workspace;              // caller scratch (NULL: no key-range splits)
  int* trace;                   // progress words in host-mapped memory (trace builds only)
};

// Query heads of one kv group that share a prefill CTA (and its K/V tiles).
inline int prefill_heads_per_cta(int n_q_heads, int n_kv_heads) {
  return ((n_q_heads / n_kv_heads) % 2 == 0) ? 2 : 1;
}
// Bytes of the prefill workspace for `hpc` heads per CTA and head_dim `d`.
size_t prefill_workspace_bytes(int hpc, int d);

// TMA descriptors of the prefill, built on the host per call.
struct PrefillMaps {
  CUtensorMap q;        // q [B][T][Hq][d]       box {d_box, 1, 128, 1}
  CUtensorMap k;        // k [B][T][Hkv][d]
  CUtensorMap v;
  CUtensorMap kc;       // k_cache [B*Hkv][W][d] box {d_box, 128, 1}
  CUtensorMap vc;
  CUtensorMap out;      // out [B][T][Hq][d] bf16, box {d_box, 1, 128, 1} (out_tma only)
};

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream);
// How a prefill launch covers its units: whole units, the split tail, the grid.
struct PrefillSchedule {
  long long n_whole;
  int n_pieces;
  long long n_items;
  int persistent;
  long long grid;
};
PrefillSchedule prefill_schedule(long long n_units, int n_wtiles, int n_sms, bool have_workspace);
int device_sm_count(int device);
cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& maps, int grid, cudaStream_t stream);
// TMA box width (elements of d per box row) and swizzle span used by the prefill kernel.
void prefill_map_geometry(int head_dim, int* box_elems, int* swizzle_bytes);

// Helpers of the C-ABI layer for entry points defined in other files: set the
// thread-local error message, look up the device status word, and run the
// host-side argument checks of a decode call (everything but the workspace).
int api_fail(int code, const char* fmt, ...);
int api_ok();
int api_status_word(int** out);
int api_check_decode(const struct swa_dims* dims, const void* out, const void* q, const void* k_new,
                     const void* v_new, const void* k_cache, const void* v_cache, const int32_t* pos);

}  // namespace swa
