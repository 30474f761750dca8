// swa_append.cu - write a chunk's keys/values into the rolling cache
// (Mistral 7B, section 2, Rolling Buffer Cache paragraph and Figure 2: the
// key/value of position i is stored in slot i mod W, overwriting older ones).
//
// Pure copy: each thread moves 16 bytes (8 bf16) of K and of V.  Source rows
// are [B][max_tokens][Hkv][d]; destination rows are [B][Hkv][W][d] at slot
// (start_pos[b] + t) mod W.  max_tokens <= W, so the slots of one call are
// distinct and the copy order does not matter.
#include "swa_common.cuh"
#include "swa_internal.h"

namespace swa {

__global__ void __launch_bounds__(256) swa_append_kernel(const AppendParams p) {
  wait_prior_grid();
  allow_next_grid();
  const int b = blockIdx.y;
  const int s0 = p.start_pos[b];
  const int n = p.n_tokens[b];
  if (s0 < 0 || n < 0 || n > p.max_tokens) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(p.status, SWA_ERR_DEVICE_ARG);
    return;
  }
  // 32-bit index arithmetic: the host keeps max_tokens * Hkv * d / 8 < 2^31,
  // and start_pos + t < 2^31 (start_pos is an int32, t < W).
  const uint32_t vecs = (uint32_t)p.head_dim / 8;       // 16-byte vectors per row
  const uint32_t per_tok = (uint32_t)p.n_kv_heads * vecs;
  const uint32_t total = (uint32_t)n * per_tok;
  const uint32_t W = (uint32_t)p.window;
  const uint4* ks = reinterpret_cast<const uint4*>(p.k) + (size_t)b * p.max_tokens * per_tok;
  const uint4* vs = reinterpret_cast<const uint4*>(p.v) + (size_t)b * p.max_tokens * per_tok;
  uint4* kd = reinterpret_cast<uint4*>(p.k_cache) + (size_t)b * p.n_kv_heads * W * vecs;
  uint4* vd = reinterpret_cast<uint4*>(p.v_cache) + (size_t)b * p.n_kv_heads * W * vecs;
  for (uint32_t e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    const uint32_t tok = e / per_tok;
    const uint32_t r = e - tok * per_tok;
    const uint32_t h = r / vecs;
    const uint32_t c = r - h * vecs;
    const uint32_t slot = ((uint32_t)s0 + tok) % W;
    const size_t dst = ((size_t)h * W + slot) * vecs + c;
    kd[dst] = ks[e];
    vd[dst] = vs[e];
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const long long per_seq = (long long)p.max_tokens * p.n_kv_heads * (p.head_dim / 8);
  long long blocks = (per_seq + 255) / 256;
  if (blocks > 1184) blocks = 1184;  // 148 SMs x 8; the kernel loops over the rest
  if (blocks < 1) blocks = 1;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, (unsigned)p.batch);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, swa_append_kernel, p);
}

}  // namespace swa
