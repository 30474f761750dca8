/*
 * swa.h - C ABI of libswa.so: sliding-window attention (SWA) with grouped-query
 * attention (GQA) over a rolling-buffer KV cache, on NVIDIA B200 (sm_100a).
 *
 * The operations follow Mistral 7B, section 2 "Architectural details":
 *   - Sliding Window Attention (paragraph, Figure 1): query position i attends
 *     to key positions j with i - W < j <= i (at most W of them).
 *   - Rolling Buffer Cache (paragraph, Figure 2): a cache of W slots per
 *     sequence and kv head; the key/value of position i live in slot i mod W.
 *   - Pre-fill and Chunking (paragraph, Figure 3): a prompt is fed in chunks of
 *     at most W tokens; each chunk attends to the cache and, causally, to itself.
 *   - Grouped-query attention (section 1): Hq / Hkv query heads share one kv
 *     head; query head h reads kv head h / (Hq / Hkv).
 *
 * Conventions for every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The library
 *     allocates no device memory and keeps no pointer after the call returns.
 *   - Tensors are dense, row-major (last index fastest), with no padding
 *     between rows; the layouts below give the index order.  bf16 means IEEE
 *     bfloat16 (torch.bfloat16).  Base pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously on it; no call synchronises the host.  Calls on
 *     one stream run in issue order.
 *   - Return value: SWA_OK, or an error code below with a message available
 *     from swa_last_error() (thread-local).  Argument errors are detected on
 *     the host before anything is launched, and then nothing is enqueued.
 *   - Integer per-sequence arguments (start_pos, n_tokens, pos) live in device
 *     memory so that calls can be captured in CUDA graphs; values the kernels
 *     find invalid there (negative positions, n_tokens > max_tokens) make the
 *     kernels skip that sequence and raise SWA_ERR_DEVICE_ARG in the device
 *     status word (swa_device_status).
 *   - Cache slots never written must hold finite values (allocate the caches
 *     zeroed): kernels read whole tiles and mask, and a NaN in a masked slot
 *     would still reach the output through 0 * NaN.
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SWA_API __attribute__((visibility("default")))
#else
#define SWA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define SWA_OK                      0
#define SWA_ERR_INVALID_ARG         1  /* null pointer, bad size, misalignment   */
#define SWA_ERR_UNSUPPORTED         2  /* head_dim not in {16,64,128}, Hq % Hkv  */
#define SWA_ERR_WORKSPACE_TOO_SMALL 3  /* swa_decode workspace below the minimum  */
#define SWA_ERR_CUDA                4  /* CUDA launch / driver error              */
#define SWA_ERR_TIMEOUT             5  /* a bounded device wait ran out           */
#define SWA_ERR_DEVICE_ARG          6  /* device-side argument out of range       */

/* Output element types. */
#define SWA_DTYPE_BF16 0
#define SWA_DTYPE_F32  1

/* Shape of one attention layer. */
typedef struct swa_dims {
    int32_t batch;       /* B: sequences                                        */
    int32_t n_q_heads;   /* Hq: query heads                                     */
    int32_t n_kv_heads;  /* Hkv: key/value heads, Hq % Hkv == 0 (G = Hq / Hkv)  */
    int32_t head_dim;    /* d: 16, 64 or 128                                    */
    int32_t window;      /* W >= 1: window length = cache slots per (seq, kv head) */
    float   scale;       /* multiplier on q.k before the softmax (e.g. 1/sqrt(d)) */
    int32_t out_dtype;   /* SWA_DTYPE_BF16 or SWA_DTYPE_F32                     */
} swa_dims;

/*
 * swa_cache_append - write a chunk's keys and values into the rolling cache.
 * Rolling Buffer Cache paragraph and Figure 2: position p goes to slot p mod W,
 * overwriting the position p - W that was there.
 *
 *   k_cache, v_cache  [B][Hkv][W][d] bf16, updated in place
 *   k, v              [B][max_tokens][Hkv][d] bf16: row t of sequence b is the
 *                     token at position start_pos[b] + t
 *   max_tokens        row capacity of k / v, 1 <= max_tokens <= W, and
 *                     max_tokens * Hkv * d / 8 < 2^31 (else SWA_ERR_UNSUPPORTED)
 *   start_pos         device int32[B], >= 0
 *   n_tokens          device int32[B], 0 <= n_tokens[b] <= max_tokens: rows
 *                     [0, n_tokens[b]) are written, the rest ignored
 * Because max_tokens <= W, no two rows of one call share a slot.
 * Must be issued after swa_prefill_chunk of the same chunk (which reads the
 * cache as it was before the chunk).
 */
SWA_API int swa_cache_append(const swa_dims* dims, void* k_cache, void* v_cache,
                     const void* k, const void* v, int32_t max_tokens,
                     const int32_t* start_pos, const int32_t* n_tokens, void* stream);

/*
 * swa_prefill_workspace_size - bytes of device scratch swa_prefill_chunk may
 * use for these dims and this max_tokens: per-row partial results of query
 * tiles whose key range is split across CTAs, and the work and merge counters.
 * Depends only on its arguments.  Returns 0 for invalid arguments.
 */
SWA_API size_t swa_prefill_workspace_size(const swa_dims* dims, int32_t max_tokens);

/*
 * swa_prefill_chunk - attention of one prefill chunk (Pre-fill and Chunking
 * paragraph, Figure 3).  Query row t of sequence b sits at position
 * i = start_pos[b] + t and attends to
 *   - the cache as it was before this chunk: the positions in
 *     [max(0, i - W + 1), start_pos[b]) it holds, and
 *   - the chunk itself, causally: rows u <= t.
 *
 *   out               [B][max_tokens][Hq][d], bf16 or f32 per dims->out_dtype;
 *                     rows t >= n_tokens[b] are not written
 *   q                 [B][max_tokens][Hq][d] bf16
 *   k, v              [B][max_tokens][Hkv][d] bf16 (the chunk's own keys/values);
 *                     rows [n_tokens[b], max_tokens) must hold finite values
 *                     (they are loaded with their tile and masked, and a NaN
 *                     there would reach the output through 0 * NaN)
 *   max_tokens        1 <= max_tokens <= W
 *   k_cache, v_cache  [B][Hkv][W][d] bf16, read only; slots must hold the
 *                     positions earlier appends put there.  A sequence whose
 *                     start_pos is 0 reads nothing from them.
 *   start_pos, n_tokens  device int32[B], as in swa_cache_append
 *   workspace         NULL (with workspace_bytes 0), or device scratch of at
 *                     least swa_prefill_workspace_size(dims, max_tokens) bytes,
 *                     16-byte aligned, ZERO-FILLED before its first use (every
 *                     call leaves it zero-filled again, so this is needed once).
 *                     With a workspace the kernel runs one CTA per SM that
 *                     takes query tiles from a shared counter and splits the
 *                     key ranges of the last tiles across CTAs (their partial
 *                     softmax results are merged by log-sum-exp); without one
 *                     it launches one CTA per query tile and head pair.  The
 *                     results agree within rounding.  Calls that may overlap
 *                     on the GPU need separate workspaces.
 * The softmax is computed in fp32 from bf16 q.k products accumulated in fp32;
 * the probabilities are rounded to bf16 for the P.V product.
 */
SWA_API int swa_prefill_chunk(const swa_dims* dims, void* out, const void* q, const void* k,
                      const void* v, int32_t max_tokens, const void* k_cache,
                      const void* v_cache, const int32_t* start_pos,
                      const int32_t* n_tokens, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * swa_decode_workspace_size - bytes of device scratch swa_decode may use for
 * these dims (fp32 partial results of a split cache sweep).  Depends only on
 * dims.  Some dims use none of it (one split per sequence and kv head, or
 * splits merged inside a thread-block cluster); the size is still reported so
 * that it stays a function of the dims.  Returns 0 for invalid dims.
 */
SWA_API size_t swa_decode_workspace_size(const swa_dims* dims);

/*
 * swa_decode_launch_info - how swa_decode runs for these dims, for callers
 * that count kernels (CUDA graphs, profilers).  Host only; enqueues nothing.
 *   n_splits    receives the number of parts the W slots of one (sequence,
 *               kv head) are split into (one CTA each)
 *   n_launches  receives the number of kernels one swa_decode call launches:
 *               1, or 2 when a combine kernel merges per-split partials
 * Either pointer may be NULL.  Returns SWA_OK, or the same codes as
 * swa_decode for invalid dims.
 */
SWA_API int swa_decode_launch_info(const swa_dims* dims, int32_t* n_splits, int32_t* n_launches);

/*
 * swa_decode - one generated token per sequence (token-by-token generation,
 * Rolling Buffer Cache paragraph).  The new key/value of position pos[b] is
 * written to slot pos[b] mod W, then the query attends over the cache: the
 * min(pos[b] + 1, W) positions (pos[b] - W, pos[b]].
 *
 *   out               [B][Hq][d], bf16 or f32 per dims->out_dtype
 *   q                 [B][Hq][d] bf16
 *   k_new, v_new      [B][Hkv][d] bf16
 *   k_cache, v_cache  [B][Hkv][W][d] bf16, slot pos[b] mod W updated in place
 *   pos               device int32[B], >= 0; the cache must hold positions
 *                     [max(0, pos[b] - W + 1), pos[b]) from earlier calls
 *   workspace         device scratch of at least swa_decode_workspace_size(dims)
 *                     bytes, 16-byte aligned; contents need no initialisation
 *                     and are garbage afterwards.  Calls that may overlap on
 *                     the GPU need separate workspaces.
 */
SWA_API int swa_decode(const swa_dims* dims, void* out, const void* q, const void* k_new,
               const void* v_new, void* k_cache, void* v_cache, const int32_t* pos,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * swa_decode_static - swa_decode for callers that cannot allocate device
 * memory.  The paper has no counterpart to this call; it exists for the
 * library's users.  Some callers cannot allocate: an engine that plans all GPU
 * memory up front and hands out only fixed buffers, or host code that gets
 * tensor pointers from a framework that owns every allocation.  Such a caller
 * passes the same inputs and outputs as to swa_decode (same meaning, layout
 * and ownership) but no workspace.
 *   - The decode scratch comes from one array built into the library,
 *     4 MiB (4194304 bytes) per device, held by every GPU that loads the
 *     library until the process exits.  A launch whose splits merge through
 *     memory needs B * Hq * n_splits * (d + 2) * 4 bytes of it (n_splits from
 *     swa_decode_launch_info; none when that reports one launch).  Dims that
 *     need more than 4 MiB are rejected with SWA_ERR_WORKSPACE_TOO_SMALL and
 *     nothing is enqueued.
 *   - The call allocates nothing.  Its first call on each device looks up the
 *     array's device address, with that device current; make that first call
 *     before any stream capture begins.
 *   - All calls on a device share the array, which keeps the previous call's
 *     contents.  Nothing in it needs clearing, because each call writes every
 *     scratch value it reads.  Calls that may overlap on the GPU (other
 *     streams, unordered host threads) race on it: order them on one stream,
 *     or use swa_decode with separate workspaces.
 */
SWA_API int swa_decode_static(const swa_dims* dims, void* out, const void* q, const void* k_new,
                      const void* v_new, void* k_cache, void* v_cache, const int32_t* pos,
                      void* stream);

/*
 * swa_device_status - synchronise `stream`, then read and clear the library's
 * device status word on the current device: SWA_OK, SWA_ERR_TIMEOUT (a
 * bounded wait inside a kernel ran out; that kernel's outputs are invalid) or
 * SWA_ERR_DEVICE_ARG.  Returns SWA_ERR_CUDA if the synchronisation fails.
 */
SWA_API int swa_device_status(void* stream);

/* Message of the last non-OK return on this thread ("" if none). */
SWA_API const char* swa_last_error(void);

/* ABI version (major * 100 + minor). */
SWA_API int swa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
