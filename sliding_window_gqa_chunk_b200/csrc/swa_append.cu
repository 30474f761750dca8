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
  const int b = blockIdx.y;
  const long long s0 = p.start_pos[b];
  const int n = p.n_tokens[b];
  if (s0 < 0 || n < 0 || n > p.max_tokens) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_status(p.status, SWA_ERR_DEVICE_ARG);
    return;
  }
  const int vecs = p.head_dim / 8;                    // 16-byte vectors per row
  const long long per_tok = (long long)p.n_kv_heads * vecs;
  const long long total = (long long)n * per_tok;
  const uint4* ks = reinterpret_cast<const uint4*>(p.k) + (long long)b * p.max_tokens * per_tok;
  const uint4* vs = reinterpret_cast<const uint4*>(p.v) + (long long)b * p.max_tokens * per_tok;
  uint4* kd = reinterpret_cast<uint4*>(p.k_cache) + (long long)b * p.n_kv_heads * p.window * vecs;
  uint4* vd = reinterpret_cast<uint4*>(p.v_cache) + (long long)b * p.n_kv_heads * p.window * vecs;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long tok = e / per_tok;
    const int r = (int)(e - tok * per_tok);
    const int h = r / vecs;
    const int c = r - h * vecs;
    const long long slot = (s0 + tok) % p.window;
    const long long dst = ((long long)h * p.window + slot) * vecs + c;
    kd[dst] = ks[e];
    vd[dst] = vs[e];
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream) {
  const long long per_seq = (long long)p.max_tokens * p.n_kv_heads * (p.head_dim / 8);
  long long blocks = (per_seq + 255) / 256;
  if (blocks > 1184) blocks = 1184;  // 148 SMs x 8; the kernel loops over the rest
  if (blocks < 1) blocks = 1;
  dim3 grid((unsigned)blocks, (unsigned)p.batch);
  swa_append_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace swa
