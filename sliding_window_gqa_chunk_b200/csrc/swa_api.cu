// swa_api.cu - the extern "C" entry points of libswa.so (declared in swa.h):
// argument validation, the thread-local error message, the per-device status
// word, TMA descriptor encoding for the prefill, and kernel dispatch.
//
// Nothing here allocates device memory.  Every check that can be made on the
// host is made before the first launch, so a call that returns an argument
// error has enqueued nothing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "swa.h"
#include "swa_internal.h"

namespace {

thread_local char g_last_error[512] = "";

// An NVTX range around each entry point, so profilers (nsys, ncu's NVTX
// filters) see the library's calls by name.  Header-only NVTX: without a
// profiler attached a push / pop is a check of a null function pointer.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
};

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_last_error[0] = '\0';
  return SWA_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SWA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- status word
// One int per device, written by kernels with atomicCAS (first error wins).
__device__ int g_swa_status;

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
int* g_status_ptr[kMaxDevices] = {};

// Device address of g_swa_status on the current device (looked up once per device).
int status_ptr(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SWA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (g_status_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_swa_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return SWA_OK;
}

// ---------------------------------------------------------------- validation
int check_dims(const swa_dims* d) {
  if (d == nullptr) return fail(SWA_ERR_INVALID_ARG, "dims is NULL");
  if (d->batch < 1 || d->batch > 65535) return fail(SWA_ERR_INVALID_ARG, "batch %d not in [1, 65535]", d->batch);
  if (d->n_q_heads < 1 || d->n_kv_heads < 1)
    return fail(SWA_ERR_INVALID_ARG, "head counts must be >= 1 (Hq=%d, Hkv=%d)", d->n_q_heads, d->n_kv_heads);
  if (d->n_q_heads % d->n_kv_heads != 0)
    return fail(SWA_ERR_UNSUPPORTED, "Hq=%d is not a multiple of Hkv=%d", d->n_q_heads, d->n_kv_heads);
  if (d->n_q_heads / d->n_kv_heads > 16)
    return fail(SWA_ERR_UNSUPPORTED, "group size Hq/Hkv=%d above 16", d->n_q_heads / d->n_kv_heads);
  if (d->n_kv_heads > 65535 || d->n_q_heads > 65535)
    return fail(SWA_ERR_INVALID_ARG, "head count above 65535");
  if (d->head_dim != 16 && d->head_dim != 64 && d->head_dim != 128)
    return fail(SWA_ERR_UNSUPPORTED, "head_dim %d not in {16, 64, 128}", d->head_dim);
  if (d->window < 1) return fail(SWA_ERR_INVALID_ARG, "window %d < 1", d->window);
  if (!(d->scale > 0.f) || !std::isfinite(d->scale))
    return fail(SWA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (d->out_dtype != SWA_DTYPE_BF16 && d->out_dtype != SWA_DTYPE_F32)
    return fail(SWA_ERR_INVALID_ARG, "out_dtype %d unknown", d->out_dtype);
  return SWA_OK;
}

int check_ptrs(const char* names, std::initializer_list<const void*> ptrs) {
  int i = 0;
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(SWA_ERR_INVALID_ARG, "pointer #%d of (%s) is NULL", i, names);
    if (!aligned16(p)) return fail(SWA_ERR_INVALID_ARG, "pointer #%d of (%s) is not 16-byte aligned", i, names);
    ++i;
  }
  return SWA_OK;
}

int check_int_ptrs(const char* names, std::initializer_list<const int32_t*> ptrs) {
  int i = 0;
  for (const int32_t* p : ptrs) {
    if (p == nullptr) return fail(SWA_ERR_INVALID_ARG, "pointer #%d of (%s) is NULL", i, names);
    if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)
      return fail(SWA_ERR_INVALID_ARG, "pointer #%d of (%s) is not 4-byte aligned", i, names);
    ++i;
  }
  return SWA_OK;
}

// ---------------------------------------------------------------- TMA encoding
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

int get_encode(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (cached == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || p == nullptr)
      return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found (%s)", cudaGetErrorName(e));
    cached = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = cached;
  return SWA_OK;
}

// rank-`rank` bf16 map, dims innermost first, byte strides of dims 1..rank-1.
int encode_map(EncodeTiledFn fn, CUtensorMap* map, const void* ptr, int rank, const cuuint64_t* dims,
               const cuuint64_t* strides, const cuuint32_t* box, int swizzle_bytes, const char* what) {
  cuuint32_t estride[5] = {1, 1, 1, 1, 1};
  CUtensorMapSwizzle swz = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                           : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                           : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(ptr), dims,
                  strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", what, (int)r);
  return SWA_OK;
}

// The TMA descriptors of a prefill call depend only on the tensors'
// addresses and the shape, so they are kept for repeated calls (a prompt's
// chunks, a decode loop that feeds one-token chunks): a small cache, replaced
// round robin, keyed by device, pointers and shape.
struct MapKey {
  int device;
  const void* ptr[6];
  int batch, n_q_heads, n_kv_heads, head_dim, window, max_tokens, out_dtype;
  bool operator==(const MapKey& o) const {
    return device == o.device && memcmp(ptr, o.ptr, sizeof(ptr)) == 0 && batch == o.batch &&
           n_q_heads == o.n_q_heads && n_kv_heads == o.n_kv_heads && head_dim == o.head_dim &&
           window == o.window && max_tokens == o.max_tokens && out_dtype == o.out_dtype;
  }
};

// Whole output tiles of the prefill go out through shared memory and a TMA
// store for bf16 output at d = 128 (the kernel has the staging buffer there).
bool prefill_out_tma(const swa_dims* dims) {
  return dims->out_dtype == SWA_DTYPE_BF16 && dims->head_dim == 128;
}
constexpr int kMapCacheSize = 16;
std::mutex g_map_mu;
MapKey g_map_keys[kMapCacheSize];
swa::PrefillMaps g_map_vals[kMapCacheSize];
int g_map_used = 0;
int g_map_next = 0;

#ifdef SWA_TEST_FAULTS
// Checked build for the host-side fault test: when set, the next descriptor
// encoding fails as if the driver had refused it (and the cache is bypassed).
int g_fail_encode = 0;
extern "C" SWA_API void swa_debug_fail_encode(int on) { g_fail_encode = on; }
#endif

int prefill_maps(int device, const swa_dims* dims, int max_tokens, const void* q, const void* k,
                 const void* v, const void* k_cache, const void* v_cache, const void* o,
                 swa::PrefillMaps* out) {
#ifdef SWA_TEST_FAULTS
  if (g_fail_encode)
    return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled(q) failed with CUresult %d (injected)",
                (int)CUDA_ERROR_INVALID_VALUE);
#endif
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.device = device;
  key.ptr[0] = q;
  key.ptr[1] = k;
  key.ptr[2] = v;
  key.ptr[3] = k_cache;
  key.ptr[4] = v_cache;
  key.ptr[5] = o;
  key.out_dtype = dims->out_dtype;
  key.batch = dims->batch;
  key.n_q_heads = dims->n_q_heads;
  key.n_kv_heads = dims->n_kv_heads;
  key.head_dim = dims->head_dim;
  key.window = dims->window;
  key.max_tokens = max_tokens;
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (int i = 0; i < g_map_used; ++i)
      if (g_map_keys[i] == key) {
        *out = g_map_vals[i];
        return SWA_OK;
      }
  }
  EncodeTiledFn enc = nullptr;
  int rc = get_encode(&enc);
  if (rc) return rc;
  const int B = dims->batch, Hq = dims->n_q_heads, Hkv = dims->n_kv_heads, D = dims->head_dim;
  const int W = dims->window;
  int box_d = 0, swz = 0;
  swa::prefill_map_geometry(D, &box_d, &swz);
  swa::PrefillMaps maps;
  memset(&maps, 0, sizeof(maps));
  const cuuint64_t es = 2;  // bf16
  {
    cuuint64_t dims4[4] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)max_tokens, (cuuint64_t)B};
    cuuint64_t str4[3] = {D * es, (cuuint64_t)Hq * D * es, (cuuint64_t)max_tokens * Hq * D * es};
    cuuint32_t box4[4] = {(cuuint32_t)box_d, 1, 128, 1};
    if ((rc = encode_map(enc, &maps.q, q, 4, dims4, str4, box4, swz, "q"))) return rc;
    // the output has the shape and element type of q
    if (prefill_out_tma(dims) && (rc = encode_map(enc, &maps.out, o, 4, dims4, str4, box4, swz, "out")))
      return rc;
  }
  {
    cuuint64_t dims4[4] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)max_tokens, (cuuint64_t)B};
    cuuint64_t str4[3] = {D * es, (cuuint64_t)Hkv * D * es, (cuuint64_t)max_tokens * Hkv * D * es};
    cuuint32_t box4[4] = {(cuuint32_t)box_d, 1, 128, 1};
    if ((rc = encode_map(enc, &maps.k, k, 4, dims4, str4, box4, swz, "k"))) return rc;
    if ((rc = encode_map(enc, &maps.v, v, 4, dims4, str4, box4, swz, "v"))) return rc;
  }
  {
    cuuint64_t dims3[3] = {(cuuint64_t)D, (cuuint64_t)W, (cuuint64_t)B * Hkv};
    cuuint64_t str3[2] = {D * es, (cuuint64_t)W * D * es};
    cuuint32_t box3[3] = {(cuuint32_t)box_d, 128, 1};
    if ((rc = encode_map(enc, &maps.kc, k_cache, 3, dims3, str3, box3, swz, "k_cache"))) return rc;
    if ((rc = encode_map(enc, &maps.vc, v_cache, 3, dims3, str3, box3, swz, "v_cache"))) return rc;
  }
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    const int i = g_map_next;
    g_map_keys[i] = key;
    g_map_vals[i] = maps;
    g_map_next = (g_map_next + 1) % kMapCacheSize;
    if (g_map_used < kMapCacheSize) ++g_map_used;
  }
  *out = maps;
  return SWA_OK;
}

// Progress words of trace builds (-DSWA_TRACE, host-mapped memory) or the tile
// counters of checked builds (-DSWA_TILE_COUNTERS, device memory), set by
// swa_debug_set_trace; always NULL in normal builds.
int* g_trace = nullptr;

}  // namespace

#if defined(SWA_TRACE) || defined(SWA_TILE_COUNTERS) || defined(SWA_TEST_FAULTS)
extern "C" SWA_API void swa_debug_set_trace(void* host_mapped) { g_trace = static_cast<int*>(host_mapped); }
#endif

namespace swa {

// Non-zero: the number of splits rounds down (at least this many), so that the
// CTAs fit in one wave of resident 4-warp CTAs (a second, nearly empty wave
// cost up to a third of the sweep); 0: rounds up.
#ifndef SWA_DECODE_SPLIT_FLOOR
#define SWA_DECODE_SPLIT_FLOOR 1
#endif

namespace {

// Resident clusters of the d = 128 stream-variant decode CTA (one per SM: a
// 192 KiB ring) on a 148-SM B200, as cudaOccupancyMaxActiveClusters reports
// them (index = cluster size): the SMs of a cluster share a GPC, so larger
// clusters leave SMs unused.  Used only where no device can be asked.
constexpr int kB200ResidentClusters[9] = {0, 148, 74, 45, 33, 26, 22, 15, 15};

int resident_clusters(int head_dim, int cs) {
  const int n = decode_resident_clusters(head_dim, cs);
  return n >= 0 ? n : kB200ResidentClusters[cs];
}

}  // namespace

DecodeSplit decode_split(int batch, int n_q_heads, int n_kv_heads, int window, int head_dim) {
  const long long units = (long long)batch * n_kv_heads;
  // Workspace split: about four resident 128-thread CTAs per SM on a 148-SM
  // B200, each split a multiple of 64 slots (16 per warp); the per-split fp32
  // partials are merged by a second kernel.  The workspace is sized for this
  // count; the launch may use fewer splits (below).
  const long long target = 148LL * 4;
  long long splits = (target + units - 1) / units;
  const long long max_splits = (window + 63) / 64;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  long long per = (window + splits - 1) / splits;
  per = (per + 63) / 64 * 64;
  DecodeSplit s;
  s.slots_per_split = (int)per;
  s.n_splits = (int)((window + per - 1) / per);
  s.ws_splits = s.n_splits;
  s.warps = 4;
  s.cluster = 0;
  s.stream = 0;
#if SWA_DECODE_SPLIT_FLOOR
  {
    long long fs = target / units;
    if (fs > max_splits) fs = max_splits;
    if (fs < SWA_DECODE_SPLIT_FLOOR) fs = SWA_DECODE_SPLIT_FLOOR;
    if (fs > splits) fs = splits;
    long long fper = (window + fs - 1) / fs;
    fper = (fper + 63) / 64 * 64;
    s.slots_per_split = (int)fper;
    s.n_splits = (int)((window + fper - 1) / fper);
  }
#endif
  if (units < 148) {
    // Fewer (sequence, kv head) pairs than SMs: one launch of CTAs whose
    // producer warp streams the split's slots into shared memory with bulk
    // copies, so every byte of a split is in flight at once.  The window of
    // a pair is split over a thread-block cluster of up to 8 CTAs (about 512
    // slots each, no more CTAs than SMs) that merge through distributed
    // shared memory; from 75 pairs on (a B200 holds 74 clusters of 2) one
    // CTA covers a pair's whole window.  No workspace and no combine kernel
    // either way.
    long long cs = 1;
    {
      // at most one CTA per SM in all (each holds a 192 KiB ring), so the
      // clusters of a launch run in one wave
      cs = (window + 511) / 512;
      if (cs > kDecodeMaxClusterSplits) cs = kDecodeMaxClusterSplits;
      if (cs > 148 / units) cs = 148 / units;
      if (cs < 1) cs = 1;
      // All clusters of the launch must be resident at once (a second wave
      // nearly doubles the step): shrink the cluster until the device holds
      // one per pair.
      while (cs > 1 && units > resident_clusters(head_dim, (int)cs)) --cs;
    }
    long long cper = (window + cs - 1) / cs;
    cper = (cper + 15) / 16 * 16;
    s.slots_per_split = (int)cper;
    s.n_splits = (int)((window + cper - 1) / cper);
    s.warps = 8;
    s.cluster = s.n_splits > 1 ? 1 : 0;
    s.stream = 1;
  }
  return s;
}

}  // namespace swa

extern "C" {

int swa_abi_version(void) { return 200; }

const char* swa_last_error(void) { return g_last_error; }

int swa_cache_append(const swa_dims* dims, void* k_cache, void* v_cache, const void* k, const void* v,
                     int32_t max_tokens, const int32_t* start_pos, const int32_t* n_tokens, void* stream) {
  CallRange range_("swa_cache_append");
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_ptrs("k_cache, v_cache, k, v", {k_cache, v_cache, k, v}))) return rc;
  if ((rc = check_int_ptrs("start_pos, n_tokens", {start_pos, n_tokens}))) return rc;
  if (max_tokens < 1 || max_tokens > dims->window)
    return fail(SWA_ERR_INVALID_ARG, "max_tokens %d not in [1, window=%d]", max_tokens, dims->window);
  if ((long long)max_tokens * dims->n_kv_heads * (dims->head_dim / 8) >= (1LL << 31))
    return fail(SWA_ERR_UNSUPPORTED, "max_tokens * Hkv * d / 8 must stay below 2^31");
  int* status = nullptr;
  if ((rc = status_ptr(&status))) return rc;
  swa::AppendParams p;
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.start_pos = start_pos;
  p.n_tokens = n_tokens;
  p.status = status;
  p.batch = dims->batch;
  p.n_kv_heads = dims->n_kv_heads;
  p.head_dim = dims->head_dim;
  p.window = dims->window;
  p.max_tokens = max_tokens;
  cudaError_t e = swa::launch_append(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "swa_cache_append launch");
  return ok();
}

size_t swa_prefill_workspace_size(const swa_dims* dims, int32_t max_tokens) {
  if (check_dims(dims) != SWA_OK) return 0;
  if (max_tokens < 1 || max_tokens > dims->window) return 0;
  const int hpc = swa::prefill_heads_per_cta(dims->n_q_heads, dims->n_kv_heads);
  return swa::prefill_workspace_bytes(hpc, dims->head_dim);
}

int swa_prefill_chunk(const swa_dims* dims, void* out, const void* q, const void* k, const void* v,
                      int32_t max_tokens, const void* k_cache, const void* v_cache, const int32_t* start_pos,
                      const int32_t* n_tokens, void* workspace, size_t workspace_bytes, void* stream) {
  CallRange range_("swa_prefill_chunk");
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_ptrs("out, q, k, v, k_cache, v_cache", {out, q, k, v, k_cache, v_cache}))) return rc;
  if ((rc = check_int_ptrs("start_pos, n_tokens", {start_pos, n_tokens}))) return rc;
  if (max_tokens < 1 || max_tokens > dims->window)
    return fail(SWA_ERR_INVALID_ARG, "max_tokens %d not in [1, window=%d]", max_tokens, dims->window);
  if (workspace == nullptr) {
    if (workspace_bytes != 0)
      return fail(SWA_ERR_INVALID_ARG, "workspace is NULL but workspace_bytes is %zu", workspace_bytes);
  } else {
    if (!aligned16(workspace)) return fail(SWA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    const size_t need = swa_prefill_workspace_size(dims, max_tokens);
    if (workspace_bytes < need)
      return fail(SWA_ERR_WORKSPACE_TOO_SMALL, "prefill workspace of %zu bytes, %zu needed", workspace_bytes,
                  need);
  }
  const int B = dims->batch, Hq = dims->n_q_heads, Hkv = dims->n_kv_heads, D = dims->head_dim;
  const int W = dims->window;
  const int hpc = swa::prefill_heads_per_cta(Hq, Hkv);
  const int n_q_tiles = (max_tokens + 127) / 128;
  const long long n_units = (long long)B * (Hq / hpc) * n_q_tiles;
  if (n_units > (1LL << 29))
    return fail(SWA_ERR_UNSUPPORTED, "%lld query tiles x head pairs in one call (limit 2^29)", n_units);
  int* status = nullptr;
  if ((rc = status_ptr(&status))) return rc;
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  swa::PrefillMaps maps;
  if ((rc = prefill_maps(device, dims, max_tokens, q, k, v, k_cache, v_cache, out, &maps))) return rc;

  const swa::PrefillSchedule sc =
      swa::prefill_schedule(n_units, (W + 127) / 128, swa::device_sm_count(device), workspace != nullptr);
  swa::PrefillParams p;
  p.out = out;
  p.start_pos = start_pos;
  p.n_tokens = n_tokens;
  p.status = status;
  p.batch = B;
  p.n_q_heads = Hq;
  p.n_kv_heads = Hkv;
  p.head_dim = D;
  p.window = W;
  p.max_tokens = max_tokens;
  p.heads_per_cta = hpc;
  p.n_q_tiles = n_q_tiles;
  p.n_whole = (int)sc.n_whole;
  p.n_pieces = sc.n_pieces;
  p.n_items = (int)sc.n_items;
  p.persistent = sc.persistent;
  p.workspace = workspace;
  p.scale_log2 = dims->scale * 1.4426950408889634f;
  p.out_f32 = dims->out_dtype == SWA_DTYPE_F32;
  // every row and 16-element piece of a row starts 32 bytes apart from the base
  p.out_v8 = (reinterpret_cast<uintptr_t>(out) % 32) == 0;
  p.out_tma = prefill_out_tma(dims) ? 1 : 0;
  p.trace = g_trace;
  e = swa::launch_prefill(p, maps, (int)sc.grid, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "swa_prefill_chunk launch");
  return ok();
}

size_t swa_decode_workspace_size(const swa_dims* dims) {
  if (check_dims(dims) != SWA_OK) return 0;
  const swa::DecodeSplit sp =
      swa::decode_split(dims->batch, dims->n_q_heads, dims->n_kv_heads, dims->window, dims->head_dim);
  if (sp.ws_splits <= 1) return 16;  // nothing needed; a non-zero size keeps callers simple
  const size_t bh = (size_t)dims->batch * dims->n_q_heads * sp.ws_splits;
  return bh * dims->head_dim * sizeof(float) + bh * 2 * sizeof(float);
}

int swa_decode_launch_info(const swa_dims* dims, int32_t* n_splits, int32_t* n_launches) {
  int rc = check_dims(dims);
  if (rc) return rc;
  const swa::DecodeSplit sp =
      swa::decode_split(dims->batch, dims->n_q_heads, dims->n_kv_heads, dims->window, dims->head_dim);
  if (n_splits) *n_splits = sp.n_splits;
  // a cluster merges its splits in-kernel; otherwise several splits need the combine kernel
  if (n_launches) *n_launches = (sp.n_splits > 1 && !sp.cluster) ? 2 : 1;
  return ok();
}

int swa_decode(const swa_dims* dims, void* out, const void* q, const void* k_new, const void* v_new,
               void* k_cache, void* v_cache, const int32_t* pos, void* workspace, size_t workspace_bytes,
               void* stream) {
  CallRange range_("swa_decode");
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_ptrs("out, q, k_new, v_new, k_cache, v_cache, workspace",
                       {out, q, k_new, v_new, k_cache, v_cache, workspace})))
    return rc;
  if ((rc = check_int_ptrs("pos", {pos}))) return rc;
  const size_t need = swa_decode_workspace_size(dims);
  if (workspace_bytes < need)
    return fail(SWA_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  int* status = nullptr;
  if ((rc = status_ptr(&status))) return rc;
  const swa::DecodeSplit sp =
      swa::decode_split(dims->batch, dims->n_q_heads, dims->n_kv_heads, dims->window, dims->head_dim);
  swa::DecodeParams p;
  p.out = out;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  p.k_cache_w = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache_w = static_cast<__nv_bfloat16*>(v_cache);
  p.pos = pos;
  const size_t bh = (size_t)dims->batch * dims->n_q_heads * sp.ws_splits;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = static_cast<float*>(workspace) + bh * dims->head_dim;
  p.status = status;
  p.batch = dims->batch;
  p.n_q_heads = dims->n_q_heads;
  p.n_kv_heads = dims->n_kv_heads;
  p.head_dim = dims->head_dim;
  p.window = dims->window;
  p.n_splits = sp.n_splits;
  p.slots_per_split = sp.slots_per_split;
  p.warps = sp.warps;
  p.cluster = sp.cluster;
  p.stream = sp.stream;
  p.scale_log2 = dims->scale * 1.4426950408889634f;
  p.out_f32 = dims->out_dtype == SWA_DTYPE_F32;
  cudaError_t e = swa::launch_decode(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "swa_decode launch");
  return ok();
}

int swa_device_status(void* stream) {
  CallRange range_("swa_device_status");
  int* status = nullptr;
  int rc = status_ptr(&status);
  if (rc) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int value = 0;
  e = cudaMemcpy(&value, status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  const int zero = 0;
  e = cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  if (value != SWA_OK) return fail(value, "device status %d raised by a kernel", value);
  return ok();
}

}  // extern "C"

// Helpers for entry points defined in other translation units.
namespace swa {

int api_fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int api_ok() { return ok(); }

int api_status_word(int** out) { return status_ptr(out); }

int api_check_decode(const swa_dims* dims, const void* out, const void* q, const void* k_new,
                     const void* v_new, const void* k_cache, const void* v_cache, const int32_t* pos) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if ((rc = check_ptrs("out, q, k_new, v_new, k_cache, v_cache", {out, q, k_new, v_new, k_cache, v_cache})))
    return rc;
  return check_int_ptrs("pos", {pos});
}

}  // namespace swa
