/*
 * videomla.h -- C ABI of the B200 (sm_100a) VideoMLA latent-KV chunk-attention library.
 *
 * Method: VideoMLA, "Low-Rank Latent KV Cache for Minute-Scale Autoregressive
 * Video Diffusion" (abstract; summary page, "Approach" and "Key results").
 * In chunk-causal autoregressive video diffusion (Wan2.1-T2V-1.3B, 12 heads of
 * 128) every cached token keeps, per layer, a head-shared content latent
 * c = x . W_DKV^T (d_c = 192) and a head-shared decoupled 3D-RoPE key
 * k_r = RoPE3D(x . W_KR^T) (d_r = 32): 224 scalars instead of 2 x 12 x 128 = 3072
 * (92.7% less).  The current chunk's queries attend to the sliding window of
 * cached frames plus the chunk itself.
 *
 * Conventions for every call
 *   - bf16 data are passed as pointers to their 16-bit patterns (uint16_t).
 *   - All tensor pointers are DEVICE pointers, contiguous row-major, 16-byte
 *     aligned.  The caller owns every buffer; the library allocates no device
 *     memory per call (its only device memory is a status word per device and
 *     the fixed scratch of vmla_chunk_attention_nonabsorbed_noalloc).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it and never synchronise, except vmla_get_device_status.
 *   - Argument errors return VMLA_ERR_INVALID_ARG / VMLA_ERR_UNSUPPORTED before
 *     anything is launched; no output is written then.  vmla_last_error()
 *     describes the most recent failure of the calling thread.
 *   - Kernels never trap.  Every internal wait has a time limit; a wait that
 *     runs out records a code that vmla_get_device_status reports.
 *   - Compiled sizes: d_c = 192 (also 64, 128, 256 through the *_dc calls),
 *     d_r = 32, per-head dim 128.  The 32 rope dims
 *     split into (t: 12, h: 10, w: 10); pair i of an axis with d_a dims turns at
 *     1e4^(-2i/d_a) radians per position; pairs are adjacent dims.
 *   - Token n of a call that starts at frame t0 on a grid_h x grid_w patch grid
 *     sits at (t0 + n / (grid_h*grid_w), (n / grid_w) % grid_h, n % grid_w);
 *     grid_h, grid_w <= 256 and a call spans at most 32 frames.
 */
#ifndef VIDEOMLA_H
#define VIDEOMLA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VMLA_OK = 0,
  VMLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size */
  VMLA_ERR_UNSUPPORTED = 2, /* size outside what the kernels are compiled for */
  VMLA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  VMLA_ERR_TIMEOUT = 4      /* a kernel wait ran out of time (reported by vmla_get_device_status) */
} vmla_status;

/* Human-readable name of a status code (static string). */
const char* vmla_status_string(int status);

/* Description of the last error returned to the calling thread (static per thread). */
const char* vmla_last_error(void);

/*
 * vmla_cache_append -- down-projection, 3D-RoPE and write into the latent cache.
 * (abstract: "shared low-rank content latent and a shared decoupled 3D-RoPE
 * positional key"; summary "Approach"; summary "Key results": 224 scalars.)
 *
 *   x      [batch, n_tok, d_model]   bf16, hidden states of the new tokens
 *   w_dkv  [192, d_model]            bf16, nn.Linear layout [out, in]
 *   w_kr   [32, d_model]             bf16
 *   cache  [batch, cap, 224]         bf16, row = [c (192) ; rotated k_r (32)]
 *
 * Token n of sample b goes to cache row (slot0 + n) mod cap of sample b (the
 * sliding window is a ring of `cap` slots; attention does not depend on slot
 * order).  Each output value is computed in fp32 with the fixed order
 *   acc = 0; for k = 0..d_model-1: acc = fl(acc + x[k]*w[k])   (exact products),
 * then, for the rope pairs (a, b): a' = fl(fl(a*cos) - fl(b*sin)),
 * b' = fl(fl(a*sin) + fl(b*cos)) with cos/sin the fp32 roundings of the fp64 libm
 * values, then rounded to bf16 (nearest even) -- so results are reproducible bit
 * for bit on any device.
 * Limits: d_model a multiple of 64 in [64, 16384]; 1 <= n_tok <= cap;
 * 0 <= slot0 < cap; t0 >= 0.
 */
vmla_status vmla_cache_append(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                              int32_t batch, int32_t n_tok, int32_t d_model, uint16_t* cache,
                              int64_t cap, int64_t slot0, int64_t t0, int32_t grid_h,
                              int32_t grid_w, void* stream);

/*
 * vmla_chunk_attention -- multi-head latent attention of one chunk over the cache.
 * (abstract and summary "Approach": per-head keys/values replaced by the shared
 * latent and rope key; summary: chunk-causal AR video diffusion.)
 *
 *   q      [batch, n_q, heads, 128]  bf16, content queries of the chunk
 *   q_rope [batch, n_q, heads, 32]   bf16, rope queries, NOT yet rotated; query i is
 *                                    rotated with the position of token i of a chunk
 *                                    starting at frame t0
 *   w_uk   [heads*128, 192]          bf16, key up-projection (row h*128+d)
 *   w_uv   [heads*128, 192]          bf16, value up-projection (row h*128+e)
 *   cache  [batch, cap, 224]         bf16, keys are rows [0, n_kv)
 *   out    [batch, n_q, heads, 128]  bf16
 *
 * Computes, for every sample b, head h and query i,
 *   out[b,i,h,:] = softmax_j( scale * ( q_h,i . W_UK_h . c_j + RoPE(q_r,h,i) . k_r,j ) )
 *                  . (c_j . W_UV_h^T)                     over all keys j in [0, n_kv)
 * i.e. every query sees every cached key and every key of its own chunk
 * (bidirectional inside the chunk).  W_UK is absorbed into the queries and
 * W_UV is applied once per query after the latent accumulation; bf16 tensor-core
 * products with fp32 accumulation.
 * Limits: 1 <= n_kv <= cap < 2^31; n_q >= 1; heads >= 1; scale > 0 and finite;
 * batch * ceil(n_q / 128) * heads * 8 < 2^31.
 */
vmla_status vmla_chunk_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                 const uint16_t* w_uv, const uint16_t* cache, int32_t batch,
                                 int32_t n_q, int32_t heads, int64_t cap, int64_t n_kv,
                                 int64_t t0, int32_t grid_h, int32_t grid_w, float scale,
                                 uint16_t* out, void* stream);

/*
 * vmla_chunk_attention_splitkv -- vmla_chunk_attention with a caller workspace that
 * lets the launch split work along the keys.  (Same computation as above; the split
 * is a scheduling choice of this library, with no counterpart on the pages.)
 *
 * The launch has one unit of work per (sample, 128-query tile, head), and one unit
 * runs on one SM at a time.  When the units do not fill the last wave of SMs, each
 * unit of that partial wave runs as `split` parts (2 <= split <= 8, each over at
 * least 32 key tiles of 128 keys, so windows under 8192 keys never split) over
 * consecutive key ranges: every part writes its
 * unnormalised latent accumulation with its running maximum and sum to the workspace,
 * and the part that finishes last rescales all parts to a common maximum, sums them
 * and applies W_UV.  split is chosen to minimise ceil(split * rest / SMs) / split,
 * the tail's length in units of one whole unit.  Results equal vmla_chunk_attention's
 * up to fp32 summation order.
 *
 * vmla_chunk_attention_splitkv_workspace_bytes -- bytes of workspace the call needs on
 * the current device for these sizes: 0 when the units fill whole waves (or a split
 * would not shorten the tail), so that the call needs no workspace; -1 on bad sizes
 * or when no device is current.
 *
 * workspace: caller-owned device memory of at least that many bytes, 16-byte aligned
 * (may be NULL when 0 bytes are needed).  Its contents on entry do not matter: the
 * call clears the arrival counters it holds with an asynchronous memset on `stream`
 * before the launch.  Calls sharing one workspace must not overlap on the GPU.
 * Errors: VMLA_ERR_INVALID_ARG when the workspace is missing or smaller than needed.
 */
int64_t vmla_chunk_attention_splitkv_workspace_bytes(int32_t batch, int32_t n_q, int32_t heads, int64_t n_kv);

vmla_status vmla_chunk_attention_splitkv(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                         const uint16_t* w_uv, const uint16_t* cache, int32_t batch, int32_t n_q,
                                         int32_t heads, int64_t cap, int64_t n_kv, int64_t t0, int32_t grid_h,
                                         int32_t grid_w, float scale, void* workspace, int64_t workspace_bytes,
                                         uint16_t* out, void* stream);

/*
 * The same two calls for another latent width d_c (summary "Key results": batch
 * headroom from 4.6x to at least 11.4x across latent budgets, 8.0x at the default
 * d_c = 192; summary "Limitations": d_c = 64 loses fine detail, so d_c trades
 * quality for efficiency).  d_c is one of 64, 128, 192, 256 (anything else returns
 * VMLA_ERR_UNSUPPORTED); the rope key stays 32 wide, so a cached row holds
 * d_c + 32 scalars:
 *   w_dkv [d_c, d_model];  w_uk, w_uv [heads*128, d_c];  cache [batch, cap, d_c + 32],
 *   row = [c (d_c) ; rotated k_r (32)].
 * Everything else -- arguments, arithmetic order of the append (bit-exact contract),
 * the attention's definition, limits and errors -- is as for vmla_cache_append and
 * vmla_chunk_attention, which are these calls with d_c = 192.
 */
vmla_status vmla_cache_append_dc(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                                 int32_t batch, int32_t n_tok, int32_t d_model, int32_t d_c, uint16_t* cache,
                                 int64_t cap, int64_t slot0, int64_t t0, int32_t grid_h,
                                 int32_t grid_w, void* stream);

vmla_status vmla_chunk_attention_dc(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                    const uint16_t* w_uv, const uint16_t* cache, int32_t batch,
                                    int32_t n_q, int32_t heads, int32_t d_c, int64_t cap, int64_t n_kv,
                                    int64_t t0, int32_t grid_h, int32_t grid_w, float scale,
                                    uint16_t* out, void* stream);

/*
 * vmla_dense_attention -- the per-head (3072-scalar) baseline layout, for comparison.
 * (summary "Key results": Self-Forcing's dense per-head KV cache, 3072 scalars/token.)
 *
 *   q    [batch, n_q, heads, d_head]   bf16
 *   k, v [batch, n_kv, heads, d_head]  bf16 (rope already applied to k)
 *   out  [batch, n_q, heads, d_head]   bf16
 * out[b,i,h,:] = softmax_j(scale * q_h,i . k_h,j) . v_h,j over j in [0, n_kv).
 * Limits: d_head == 128; n_kv >= 1; n_q >= 1; heads >= 1.
 */
vmla_status vmla_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 int32_t batch, int32_t n_q, int64_t n_kv, int32_t heads,
                                 int32_t d_head, float scale, uint16_t* out, void* stream);

/*
 * The projections either side of the attention (summary "Approach": the latent
 * attention block of the Wan2.1 backbone; the pages give no formulas, these are the
 * standard linear maps).  bf16 tensor-core GEMMs with fp32 accumulation, bf16 out.
 *
 * vmla_query_projection -- one pass over the hidden states x[batch, n_tok, d_model]:
 *   q      [batch, n_tok, heads, 128] = x . W_Q^T,  w_q  [heads*128, d_model]
 *   q_rope [batch, n_tok, heads, 32]  = x . W_QR^T, w_qr [heads*32, d_model]
 *   (q_rope is left unrotated: vmla_chunk_attention rotates it with the token positions.)
 *   Limits: d_model a multiple of 64; batch*n_tok < 2^31.
 *
 * vmla_output_projection -- y[batch, n_tok, d_model] = o . W_O^T with o the attention
 *   output [batch, n_tok, heads, 128] and w_o [d_model, heads*128].
 *   Limits: d_model a multiple of 128; batch*n_tok < 2^31.
 */
vmla_status vmla_query_projection(const uint16_t* x, const uint16_t* w_q, const uint16_t* w_qr, int32_t batch,
                                  int32_t n_tok, int32_t d_model, int32_t heads, uint16_t* q, uint16_t* q_rope,
                                  void* stream);

vmla_status vmla_output_projection(const uint16_t* o, const uint16_t* w_o, int32_t batch, int32_t n_tok,
                                   int32_t heads, int32_t d_model, uint16_t* y, void* stream);

/*
 * Non-absorbed form of the same attention (the latent cache stays the only cache).
 * (abstract: per-head keys and values are generated from the head-shared content
 * latent; summary "Approach".)  Per-head keys K_h = c . W_UK_h^T and values
 * V_h = c . W_UV_h^T are materialised from the cache, then each query attends with
 * the 160-dim key [K_h ; k_r] (k_r read from the cache) and the 128-dim value V_h.
 * The result equals vmla_chunk_attention's up to rounding; the work per query, head
 * and key is 2 x (160 + 128) FLOPs instead of 2 x (224 + 192), and the
 * materialisation can be shared by every denoising step of a chunk.
 *
 * vmla_materialized_kv_bytes -- bytes of the materialised buffer kv[batch, n_kv, 2*heads, 128]
 *   (bf16; heads [0, heads) hold K_h, heads [heads, 2*heads) hold V_h); 0 on bad sizes and
 *   on sizes whose byte count does not fit in int64.
 *
 * vmla_materialize_kv -- writes kv (caller-owned, vmla_materialized_kv_bytes bytes) from
 *   cache rows [0, n_kv) of cache[batch, cap, 224] and w_uk, w_uv [heads*128, 192].
 *   bf16 tensor-core products, fp32 accumulation, bf16 rounding.  Limits: 1 <= n_kv <= cap < 2^31.
 *
 * vmla_chunk_attention_materialized -- out[batch, n_q, heads, 128] from q, q_rope (as for
 *   vmla_chunk_attention), the materialised kv and the rope keys of cache rows [0, n_kv).
 *
 * vmla_chunk_attention_nonabsorbed -- both steps in one call; `workspace` (device,
 *   16-byte aligned, >= vmla_materialized_kv_bytes(batch, heads, n_kv) bytes) receives kv.
 */
int64_t vmla_materialized_kv_bytes(int32_t batch, int32_t heads, int64_t n_kv);

vmla_status vmla_materialize_kv(const uint16_t* w_uk, const uint16_t* w_uv, const uint16_t* cache,
                                int32_t batch, int32_t heads, int64_t cap, int64_t n_kv, uint16_t* kv,
                                void* stream);

vmla_status vmla_chunk_attention_materialized(const uint16_t* q, const uint16_t* q_rope, const uint16_t* kv,
                                              const uint16_t* cache, int32_t batch, int32_t n_q, int32_t heads,
                                              int64_t cap, int64_t n_kv, int64_t t0, int32_t grid_h,
                                              int32_t grid_w, float scale, uint16_t* out, void* stream);

vmla_status vmla_chunk_attention_nonabsorbed(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                             const uint16_t* w_uv, const uint16_t* cache, int32_t batch,
                                             int32_t n_q, int32_t heads, int64_t cap, int64_t n_kv, int64_t t0,
                                             int32_t grid_h, int32_t grid_w, float scale, void* workspace,
                                             int64_t workspace_bytes, uint16_t* out, void* stream);

/*
 * vmla_chunk_attention_nonabsorbed_noalloc -- vmla_chunk_attention_nonabsorbed without
 * a caller workspace: the library's own fixed scratch holds the materialised keys and
 * values.  (No counterpart in the paper: this is an interface for callers that cannot
 * allocate device memory -- for example a host program that only receives tensors from
 * another runtime, a framework whose allocator already owns the device memory budget,
 * or a loop that cannot take the device-wide synchronisation cudaMalloc/cudaFree imply.)
 *
 * Arguments and result are those of vmla_chunk_attention_nonabsorbed.  The scratch is a
 * static device array of VMLA_NOALLOC_SCRATCH_BYTES that every GPU loading the library
 * keeps until exit; sizes with vmla_materialized_kv_bytes(batch, heads, n_kv) above it
 * return VMLA_ERR_UNSUPPORTED (use the workspace form).  The call allocates nothing.
 * Its first call on a device looks up the scratch's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any stream
 * capture.  All calls on a device share the one scratch and it keeps the last call's
 * contents (nothing in it needs to start at zero), so calls that overlap on the GPU
 * -- e.g. on two streams at once -- race with each other and must be serialised.
 */
#define VMLA_NOALLOC_SCRATCH_BYTES (8ll << 20)
vmla_status vmla_chunk_attention_nonabsorbed_noalloc(const uint16_t* q, const uint16_t* q_rope,
                                                     const uint16_t* w_uk, const uint16_t* w_uv,
                                                     const uint16_t* cache, int32_t batch, int32_t n_q,
                                                     int32_t heads, int64_t cap, int64_t n_kv, int64_t t0,
                                                     int32_t grid_h, int32_t grid_w, float scale, uint16_t* out,
                                                     void* stream);

/*
 * vmla_get_device_status -- synchronises `stream`, then reports (and clears) any
 * wait timeout recorded by this library's kernels on the current device since the
 * last call: VMLA_ERR_TIMEOUT, VMLA_ERR_CUDA on a CUDA error, else VMLA_OK.
 */
vmla_status vmla_get_device_status(void* stream);

/*
 * vmla_selftest_wait_timeout -- launches one tiny kernel that waits on a barrier
 * nothing will ever complete, with a limit of `limit_ns` nanoseconds (1e3 .. 1e10).
 * The kernel gives up, records a timeout and returns, leaving the context usable;
 * a following vmla_get_device_status(stream) returns VMLA_ERR_TIMEOUT.  For tests
 * of the failure path.
 */
vmla_status vmla_selftest_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VIDEOMLA_H */
