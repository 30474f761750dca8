// swa_decode_static.cu - swa_decode_static(): the decode step of swa_decode,
// for callers that cannot hand the library a device workspace.
//
// Some callers cannot allocate device memory at all.  One example is an engine
// that plans every byte of GPU memory up front and hands out only fixed
// buffers.  Another is host code that receives tensor pointers from a
// framework that owns all allocation and gives out no allocator.  Such
// callers can still provide the inputs and outputs but have nowhere to get
// the decode's scratch from, and cudaMalloc/cudaFree would also stall the
// device in the middle of a token loop.  This entry point therefore takes its
// scratch from one array compiled into the library.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes
// (4 MiB).  Every GPU that loads the library holds its own copy until the
// process exits.  The entry point itself allocates nothing: no cudaMalloc, no
// cudaFree, no allocating library routine.
//
// Host code cannot use the array's name as a device address (on the host the
// name denotes a host-side shadow).  So on the first call on each device,
// with that device current, we ask the runtime for its device address with
// cudaGetSymbolAddress and keep it for later calls.  That first call on a
// device should therefore come before any stream capture begins.
//
// Sharing rules:
//   * every call on a device uses the same array, which keeps whatever the
//     previous call left in it;
//   * the decode writes every scratch element it reads later in the same call
//     (per-split partial maxima, sums and outputs), so nothing needs clearing;
//   * calls that may run at the same time on the GPU (different streams, or
//     host threads without ordering between them) race on the array and give
//     wrong results; order them on one stream or use swa_decode with separate
//     workspaces.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <mutex>

#include "swa.h"
#include "swa_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB, same on every device

// The decode's scratch for swa_decode_static: fp32 partials, 256-byte aligned.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// NVTX range around the entry point (see swa_api.cu).
struct StaticCallRange {
  StaticCallRange() { nvtxRangePushA("swa_decode_static"); }
  ~StaticCallRange() { nvtxRangePop(); }
};

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device; looked up once
// per device on that device's first call.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return swa::api_fail(SWA_ERR_CUDA, "cudaGetDevice failed (%s)", cudaGetErrorName(e));
  if (dev < 0 || dev >= kMaxDevices)
    return swa::api_fail(SWA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_decode_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return swa::api_fail(SWA_ERR_CUDA, "cudaGetSymbolAddress(decode scratch) failed (%s)",
                           cudaGetErrorName(e));
    g_scratch_dev[dev] = ptr;
  }
  *out = g_scratch_dev[dev];
  return SWA_OK;
}

}  // namespace

extern "C" SWA_API int swa_decode_static(const swa_dims* dims, void* out, const void* q, const void* k_new,
                                         const void* v_new, void* k_cache, void* v_cache, const int32_t* pos,
                                         void* stream) {
  StaticCallRange range_;
  int rc = swa::api_check_decode(dims, out, q, k_new, v_new, k_cache, v_cache, pos);
  if (rc) return rc;
  // The scratch this launch really uses: none when one split covers the window
  // or a thread-block cluster merges the splits, else one fp32 partial
  // (d values, max and sum) per (sequence, query head, split).
  const swa::DecodeSplit sp =
      swa::decode_split(dims->batch, dims->n_q_heads, dims->n_kv_heads, dims->window, dims->head_dim);
  const size_t bh = (size_t)dims->batch * dims->n_q_heads * sp.n_splits;
  const size_t need = (sp.cluster || sp.n_splits == 1) ? 0 : bh * (dims->head_dim + 2) * sizeof(float);
  if (need > kStaticScratchBytes)
    return swa::api_fail(SWA_ERR_WORKSPACE_TOO_SMALL,
                         "swa_decode_static: these dims need %zu bytes of decode scratch but the "
                         "built-in scratch holds %zu; call swa_decode with a workspace instead",
                         need, kStaticScratchBytes);
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch))) return rc;
  int* status = nullptr;
  if ((rc = swa::api_status_word(&status))) return rc;

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
  p.ws_o = static_cast<float*>(scratch);
  p.ws_ml = static_cast<float*>(scratch) + bh * dims->head_dim;
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
  if (e != cudaSuccess)
    return swa::api_fail(SWA_ERR_CUDA, "swa_decode_static launch: %s (%s)", cudaGetErrorName(e),
                         cudaGetErrorString(e));
  return swa::api_ok();
}
