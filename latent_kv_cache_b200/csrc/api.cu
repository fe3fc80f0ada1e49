// C ABI of the library (declared in include/videomla.h): argument validation,
// error reporting and dispatch to the kernels.  Nothing here allocates device
// memory; every tensor belongs to the caller.
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "common.cuh"
#include "videomla.h"

namespace vmla {
cudaError_t launch_cache_append(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                                int batch, int n_tok, int d_model, int d_c, uint16_t* cache, int64_t cap,
                                int64_t slot0, int64_t t0, int grid_h, int grid_w, cudaStream_t stream);
cudaError_t launch_chunk_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                   const uint16_t* w_uv, const uint16_t* cache, int batch, int n_q,
                                   int heads, int d_c, int64_t cap, int64_t n_kv, int64_t t0, int grid_h,
                                   int grid_w, float scale, uint16_t* out, int* status,
                                   cudaStream_t stream, bool* encode_failed, const SplitPlan& plan,
                                   void* workspace);
cudaError_t launch_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int batch,
                                   int n_q, int64_t n_kv, int heads, float scale, uint16_t* out,
                                   int* status, cudaStream_t stream, bool* encode_failed);
cudaError_t launch_selftest_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_materialize_kv(const uint16_t* w_uk, const uint16_t* w_uv, const uint16_t* cache, int batch,
                                  int heads, int64_t cap, int64_t n_kv, uint16_t* kv, int* status,
                                  cudaStream_t stream, bool* encode_failed);
cudaError_t launch_gemm_pair(const uint16_t* a, const uint16_t* b0, const uint16_t* b1, int m, int n0, int n1,
                             int k, uint16_t* c0, int64_t ldc0, uint16_t* c1, int64_t ldc1, int* status,
                             cudaStream_t stream, bool* encode_failed);
cudaError_t launch_mat_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* kv,
                                 const uint16_t* cache, int batch, int n_q, int heads, int64_t cap,
                                 int64_t n_kv, int64_t t0, int grid_h, int grid_w, float scale, uint16_t* out,
                                 int* status, cudaStream_t stream, bool* encode_failed);
}  // namespace vmla

namespace {

thread_local char g_last_error[512] = "no error";

vmla_status fail(vmla_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return s;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

vmla_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VMLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Common checks of the rotary-position arguments of a call covering n_tok tokens.
vmla_status check_positions(int64_t n_tok, int64_t t0, int32_t grid_h, int32_t grid_w) {
  if (grid_h < 1 || grid_w < 1) return fail(VMLA_ERR_INVALID_ARG, "grid_h/grid_w must be >= 1");
  if (grid_h > vmla::kMaxSide || grid_w > vmla::kMaxSide)
    return fail(VMLA_ERR_UNSUPPORTED, "grid_h/grid_w must be <= %d", vmla::kMaxSide);
  if (t0 < 0) return fail(VMLA_ERR_INVALID_ARG, "t0 must be >= 0");
  const int64_t per = (int64_t)grid_h * grid_w;
  if ((n_tok + per - 1) / per > vmla::kMaxFrames)
    return fail(VMLA_ERR_UNSUPPORTED, "a call may span at most %d frames", vmla::kMaxFrames);
  return VMLA_OK;
}

}  // namespace

namespace vmla {
// Sets the calling thread's vmla_last_error() message (for entry points in other files).
vmla_status record_error(vmla_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace vmla

extern "C" {

const char* vmla_status_string(int status) {
  switch (status) {
    case VMLA_OK: return "VMLA_OK";
    case VMLA_ERR_INVALID_ARG: return "VMLA_ERR_INVALID_ARG";
    case VMLA_ERR_UNSUPPORTED: return "VMLA_ERR_UNSUPPORTED";
    case VMLA_ERR_CUDA: return "VMLA_ERR_CUDA";
    case VMLA_ERR_TIMEOUT: return "VMLA_ERR_TIMEOUT";
    default: return "VMLA_ERR_UNKNOWN";
  }
}

const char* vmla_last_error(void) { return g_last_error; }

static bool supported_dc(int32_t d_c) { return d_c == 64 || d_c == 128 || d_c == 192 || d_c == 256; }

vmla_status vmla_cache_append_dc(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                                 int32_t batch, int32_t n_tok, int32_t d_model, int32_t d_c, uint16_t* cache,
                                 int64_t cap, int64_t slot0, int64_t t0, int32_t grid_h,
                                 int32_t grid_w, void* stream) {
  if (!supported_dc(d_c)) return fail(VMLA_ERR_UNSUPPORTED, "cache_append: d_c must be 64, 128, 192 or 256");
  if (!aligned16(x) || !aligned16(w_dkv) || !aligned16(w_kr) || !aligned16(cache))
    return fail(VMLA_ERR_INVALID_ARG, "cache_append: pointers must be non-null and 16-byte aligned");
  if (batch < 1 || batch > 65535) return fail(VMLA_ERR_INVALID_ARG, "cache_append: batch must be in [1, 65535]");
  if (n_tok < 1) return fail(VMLA_ERR_INVALID_ARG, "cache_append: n_tok must be >= 1");
  if (d_model < 64 || d_model > 16384 || d_model % 64 != 0)
    return fail(VMLA_ERR_UNSUPPORTED, "cache_append: d_model must be a multiple of 64 in [64, 16384]");
  if (cap < 1 || n_tok > cap) return fail(VMLA_ERR_INVALID_ARG, "cache_append: need 1 <= n_tok <= cap");
  if (slot0 < 0 || slot0 >= cap) return fail(VMLA_ERR_INVALID_ARG, "cache_append: need 0 <= slot0 < cap");
  vmla_status st = check_positions(n_tok, t0, grid_h, grid_w);
  if (st != VMLA_OK) return st;
  cudaError_t e = vmla::launch_cache_append(x, w_dkv, w_kr, batch, n_tok, d_model, d_c, cache, cap, slot0,
                                            t0, grid_h, grid_w, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cache_append launch");
  return VMLA_OK;
}

vmla_status vmla_cache_append(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                              int32_t batch, int32_t n_tok, int32_t d_model, uint16_t* cache,
                              int64_t cap, int64_t slot0, int64_t t0, int32_t grid_h,
                              int32_t grid_w, void* stream) {
  return vmla_cache_append_dc(x, w_dkv, w_kr, batch, n_tok, d_model, vmla::kDc, cache, cap, slot0, t0, grid_h,
                              grid_w, stream);
}

}  // extern "C"

namespace {

// Units of the latent attention launch: (sample, query tile, head).
int64_t latent_units(int32_t batch, int32_t n_q, int32_t heads) {
  return (int64_t)batch * ((n_q + 127) / 128) * heads;
}

// Shared body of the latent-attention entry points.  split: may run the last
// partial wave's units as key-range parts merged through `workspace`.
vmla_status chunk_attention_impl(const char* who, const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                 const uint16_t* w_uv, const uint16_t* cache, int32_t batch, int32_t n_q,
                                 int32_t heads, int32_t d_c, int64_t cap, int64_t n_kv, int64_t t0, int32_t grid_h,
                                 int32_t grid_w, float scale, bool split, void* workspace, int64_t workspace_bytes,
                                 uint16_t* out, void* stream) {
  if (!supported_dc(d_c)) return fail(VMLA_ERR_UNSUPPORTED, "%s: d_c must be 64, 128, 192 or 256", who);
  if (!aligned16(q) || !aligned16(q_rope) || !aligned16(w_uk) || !aligned16(w_uv) ||
      !aligned16(cache) || !aligned16(out))
    return fail(VMLA_ERR_INVALID_ARG, "%s: pointers must be non-null and 16-byte aligned", who);
  if (batch < 1 || batch > 65535) return fail(VMLA_ERR_INVALID_ARG, "%s: batch must be in [1, 65535]", who);
  if (n_q < 1) return fail(VMLA_ERR_INVALID_ARG, "%s: n_q must be >= 1", who);
  if (heads < 1 || heads > 512) return fail(VMLA_ERR_INVALID_ARG, "%s: heads must be in [1, 512]", who);
  if (n_kv < 1 || n_kv > cap) return fail(VMLA_ERR_INVALID_ARG, "%s: need 1 <= n_kv <= cap", who);
  if (cap >= (int64_t(1) << 31)) return fail(VMLA_ERR_UNSUPPORTED, "%s: cap must be < 2^31", who);
  if (latent_units(batch, n_q, heads) * vmla::kMaxSplit > 0x7FFFFFFF)
    return fail(VMLA_ERR_UNSUPPORTED, "%s: too many query tiles x heads x samples", who);
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VMLA_ERR_INVALID_ARG, "%s: scale must be positive and finite", who);
  vmla_status st = check_positions(n_q, t0, grid_h, grid_w);
  if (st != VMLA_OK) return st;
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "%s: no CUDA device", who);
  const int64_t units = latent_units(batch, n_q, heads);
  vmla::SplitPlan plan{units, 1, 0};
  if (split) {
    plan = vmla::plan_split(units, (int)((n_kv + 127) / 128), vmla::sm_count_current_device());
    const int64_t need = vmla::split_workspace_bytes(plan, d_c);
    if (need > 0) {
      if (!aligned16(workspace))
        return fail(VMLA_ERR_INVALID_ARG, "%s: workspace must be non-null and 16-byte aligned", who);
      if (workspace_bytes < need)
        return fail(VMLA_ERR_INVALID_ARG, "%s: workspace of %lld bytes, need %lld", who, (long long)workspace_bytes,
                    (long long)need);
    }
  }
  bool enc_fail = false;
  cudaError_t e = vmla::launch_chunk_attention(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, d_c, cap,
                                               n_kv, t0, grid_h, grid_w, scale, out, status,
                                               static_cast<cudaStream_t>(stream), &enc_fail, plan, workspace);
  if (enc_fail) return fail(VMLA_ERR_CUDA, "%s: tensor-map encoding failed", who);
  if (e != cudaSuccess) return cuda_fail(e, "chunk_attention launch");
  return VMLA_OK;
}

}  // namespace

extern "C" {

vmla_status vmla_chunk_attention_dc(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                    const uint16_t* w_uv, const uint16_t* cache, int32_t batch,
                                    int32_t n_q, int32_t heads, int32_t d_c, int64_t cap, int64_t n_kv,
                                    int64_t t0, int32_t grid_h, int32_t grid_w, float scale,
                                    uint16_t* out, void* stream) {
  return chunk_attention_impl("chunk_attention", q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, d_c, cap, n_kv,
                              t0, grid_h, grid_w, scale, false, nullptr, 0, out, stream);
}

vmla_status vmla_chunk_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                 const uint16_t* w_uv, const uint16_t* cache, int32_t batch,
                                 int32_t n_q, int32_t heads, int64_t cap, int64_t n_kv,
                                 int64_t t0, int32_t grid_h, int32_t grid_w, float scale,
                                 uint16_t* out, void* stream) {
  return vmla_chunk_attention_dc(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, vmla::kDc, cap, n_kv, t0,
                                 grid_h, grid_w, scale, out, stream);
}

int64_t vmla_chunk_attention_splitkv_workspace_bytes(int32_t batch, int32_t n_q, int32_t heads, int64_t n_kv) {
  if (batch < 1 || batch > 65535 || n_q < 1 || heads < 1 || heads > 512 || n_kv < 1 || n_kv >= (int64_t(1) << 31))
    return -1;
  if (latent_units(batch, n_q, heads) * vmla::kMaxSplit > 0x7FFFFFFF) return -1;
  const int sms = vmla::sm_count_current_device();
  if (sms <= 0) return -1;
  const vmla::SplitPlan plan =
      vmla::plan_split(latent_units(batch, n_q, heads), (int)((n_kv + 127) / 128), sms);
  return vmla::split_workspace_bytes(plan, vmla::kDc);
}

vmla_status vmla_chunk_attention_splitkv(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                         const uint16_t* w_uv, const uint16_t* cache, int32_t batch, int32_t n_q,
                                         int32_t heads, int64_t cap, int64_t n_kv, int64_t t0, int32_t grid_h,
                                         int32_t grid_w, float scale, void* workspace, int64_t workspace_bytes,
                                         uint16_t* out, void* stream) {
  return chunk_attention_impl("chunk_attention_splitkv", q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, vmla::kDc,
                              cap, n_kv, t0, grid_h, grid_w, scale, true, workspace, workspace_bytes, out, stream);
}

vmla_status vmla_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 int32_t batch, int32_t n_q, int64_t n_kv, int32_t heads,
                                 int32_t d_head, float scale, uint16_t* out, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(VMLA_ERR_INVALID_ARG, "dense_attention: pointers must be non-null and 16-byte aligned");
  if (d_head != vmla::kDh) return fail(VMLA_ERR_UNSUPPORTED, "dense_attention: d_head must be 128");
  if (batch < 1 || batch > 65535) return fail(VMLA_ERR_INVALID_ARG, "dense_attention: batch must be in [1, 65535]");
  if (n_q < 1) return fail(VMLA_ERR_INVALID_ARG, "dense_attention: n_q must be >= 1");
  if (heads < 1 || heads > 512) return fail(VMLA_ERR_INVALID_ARG, "dense_attention: heads must be in [1, 512]");
  if (n_kv < 1 || n_kv >= (int64_t(1) << 31))
    return fail(VMLA_ERR_INVALID_ARG, "dense_attention: need 1 <= n_kv < 2^31");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VMLA_ERR_INVALID_ARG, "dense_attention: scale must be positive and finite");
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "dense_attention: no CUDA device");
  bool enc_fail = false;
  cudaError_t e = vmla::launch_dense_attention(q, k, v, batch, n_q, n_kv, heads, scale, out, status,
                                               static_cast<cudaStream_t>(stream), &enc_fail);
  if (enc_fail) return fail(VMLA_ERR_CUDA, "dense_attention: tensor-map encoding failed");
  if (e != cudaSuccess) return cuda_fail(e, "dense_attention launch");
  return VMLA_OK;
}

// Shared checks of the latent-attention arguments (chunk attention, both forms).
static vmla_status check_latent_attention(const char* who, int32_t batch, int32_t n_q, int32_t heads, int64_t cap,
                                          int64_t n_kv, int64_t t0, int32_t grid_h, int32_t grid_w, float scale) {
  if (batch < 1 || batch > 65535) return fail(VMLA_ERR_INVALID_ARG, "%s: batch must be in [1, 65535]", who);
  if (n_q < 1) return fail(VMLA_ERR_INVALID_ARG, "%s: n_q must be >= 1", who);
  if (heads < 1 || heads > 512) return fail(VMLA_ERR_INVALID_ARG, "%s: heads must be in [1, 512]", who);
  if (n_kv < 1 || n_kv > cap) return fail(VMLA_ERR_INVALID_ARG, "%s: need 1 <= n_kv <= cap", who);
  if (cap >= (int64_t(1) << 31)) return fail(VMLA_ERR_UNSUPPORTED, "%s: cap must be < 2^31", who);
  if ((int64_t)((n_q + 127) / 128) * heads > 0x7FFFFFFF)
    return fail(VMLA_ERR_UNSUPPORTED, "%s: too many query tiles", who);
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VMLA_ERR_INVALID_ARG, "%s: scale must be positive and finite", who);
  return check_positions(n_q, t0, grid_h, grid_w);
}

int64_t vmla_materialized_kv_bytes(int32_t batch, int32_t heads, int64_t n_kv) {
  if (batch < 1 || heads < 1 || n_kv < 1) return 0;
  // batch * heads * 512 < 2^31 * 2^31 * 2^9 does not fit either, so divide step by step.
  const int64_t per_key = (int64_t)heads * 2 * vmla::kDh * 2;  // <= 2^31 * 512
  if ((int64_t)batch > INT64_MAX / per_key) return 0;
  const int64_t per_row = (int64_t)batch * per_key;
  if (n_kv > INT64_MAX / per_row) return 0;
  return n_kv * per_row;
}

vmla_status vmla_materialize_kv(const uint16_t* w_uk, const uint16_t* w_uv, const uint16_t* cache,
                                int32_t batch, int32_t heads, int64_t cap, int64_t n_kv, uint16_t* kv,
                                void* stream) {
  if (!aligned16(w_uk) || !aligned16(w_uv) || !aligned16(cache) || !aligned16(kv))
    return fail(VMLA_ERR_INVALID_ARG, "materialize_kv: pointers must be non-null and 16-byte aligned");
  if (batch < 1 || batch > 65535) return fail(VMLA_ERR_INVALID_ARG, "materialize_kv: batch must be in [1, 65535]");
  if (heads < 1 || heads > 512) return fail(VMLA_ERR_INVALID_ARG, "materialize_kv: heads must be in [1, 512]");
  if (n_kv < 1 || n_kv > cap) return fail(VMLA_ERR_INVALID_ARG, "materialize_kv: need 1 <= n_kv <= cap");
  if (cap >= (int64_t(1) << 31)) return fail(VMLA_ERR_UNSUPPORTED, "materialize_kv: cap must be < 2^31");
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "materialize_kv: no CUDA device");
  bool enc_fail = false;
  cudaError_t e = vmla::launch_materialize_kv(w_uk, w_uv, cache, batch, heads, cap, n_kv, kv, status,
                                              static_cast<cudaStream_t>(stream), &enc_fail);
  if (enc_fail) return fail(VMLA_ERR_CUDA, "materialize_kv: tensor-map encoding failed");
  if (e != cudaSuccess) return cuda_fail(e, "materialize_kv launch");
  return VMLA_OK;
}

vmla_status vmla_chunk_attention_materialized(const uint16_t* q, const uint16_t* q_rope, const uint16_t* kv,
                                              const uint16_t* cache, int32_t batch, int32_t n_q, int32_t heads,
                                              int64_t cap, int64_t n_kv, int64_t t0, int32_t grid_h,
                                              int32_t grid_w, float scale, uint16_t* out, void* stream) {
  if (!aligned16(q) || !aligned16(q_rope) || !aligned16(kv) || !aligned16(cache) || !aligned16(out))
    return fail(VMLA_ERR_INVALID_ARG,
                "chunk_attention_materialized: pointers must be non-null and 16-byte aligned");
  vmla_status st = check_latent_attention("chunk_attention_materialized", batch, n_q, heads, cap, n_kv, t0,
                                          grid_h, grid_w, scale);
  if (st != VMLA_OK) return st;
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "chunk_attention_materialized: no CUDA device");
  bool enc_fail = false;
  cudaError_t e = vmla::launch_mat_attention(q, q_rope, kv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                             grid_w, scale, out, status, static_cast<cudaStream_t>(stream),
                                             &enc_fail);
  if (enc_fail) return fail(VMLA_ERR_CUDA, "chunk_attention_materialized: tensor-map encoding failed");
  if (e != cudaSuccess) return cuda_fail(e, "chunk_attention_materialized launch");
  return VMLA_OK;
}

vmla_status vmla_chunk_attention_nonabsorbed(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                             const uint16_t* w_uv, const uint16_t* cache, int32_t batch,
                                             int32_t n_q, int32_t heads, int64_t cap, int64_t n_kv, int64_t t0,
                                             int32_t grid_h, int32_t grid_w, float scale, void* workspace,
                                             int64_t workspace_bytes, uint16_t* out, void* stream) {
  if (!aligned16(workspace))
    return fail(VMLA_ERR_INVALID_ARG, "chunk_attention_nonabsorbed: workspace must be non-null and 16-byte aligned");
  vmla_status st = check_latent_attention("chunk_attention_nonabsorbed", batch, n_q, heads, cap, n_kv, t0,
                                          grid_h, grid_w, scale);
  if (st != VMLA_OK) return st;
  const int64_t need = vmla_materialized_kv_bytes(batch, heads, n_kv);
  if (need <= 0)
    return fail(VMLA_ERR_UNSUPPORTED, "chunk_attention_nonabsorbed: workspace size overflows int64");
  if (workspace_bytes < need)
    return fail(VMLA_ERR_INVALID_ARG, "chunk_attention_nonabsorbed: workspace of %lld bytes, need %lld",
                (long long)workspace_bytes, (long long)need);
  uint16_t* kv = static_cast<uint16_t*>(workspace);
  st = vmla_materialize_kv(w_uk, w_uv, cache, batch, heads, cap, n_kv, kv, stream);
  if (st != VMLA_OK) return st;
  return vmla_chunk_attention_materialized(q, q_rope, kv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h, grid_w,
                                           scale, out, stream);
}

vmla_status vmla_query_projection(const uint16_t* x, const uint16_t* w_q, const uint16_t* w_qr, int32_t batch,
                                  int32_t n_tok, int32_t d_model, int32_t heads, uint16_t* q, uint16_t* q_rope,
                                  void* stream) {
  if (!aligned16(x) || !aligned16(w_q) || !aligned16(w_qr) || !aligned16(q) || !aligned16(q_rope))
    return fail(VMLA_ERR_INVALID_ARG, "query_projection: pointers must be non-null and 16-byte aligned");
  if (batch < 1 || n_tok < 1 || (int64_t)batch * n_tok > 0x7FFFFFFF)
    return fail(VMLA_ERR_INVALID_ARG, "query_projection: need batch, n_tok >= 1 and batch*n_tok < 2^31");
  if (heads < 1 || heads > 512) return fail(VMLA_ERR_INVALID_ARG, "query_projection: heads must be in [1, 512]");
  if (d_model < 64 || d_model > 65536 || d_model % 64 != 0)
    return fail(VMLA_ERR_UNSUPPORTED, "query_projection: d_model must be a multiple of 64 in [64, 65536]");
  if (((int64_t)batch * n_tok + 255) / 256 * ((heads * (vmla::kDh + vmla::kDr) + 255) / 256) > 0x7FFFFFFF)
    return fail(VMLA_ERR_UNSUPPORTED, "query_projection: more than 2^31 - 1 output tiles");
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "query_projection: no CUDA device");
  bool enc_fail = false;
  cudaError_t e = vmla::launch_gemm_pair(x, w_q, w_qr, batch * n_tok, heads * vmla::kDh, heads * vmla::kDr, d_model,
                                         q, (int64_t)heads * vmla::kDh, q_rope, (int64_t)heads * vmla::kDr, status,
                                         static_cast<cudaStream_t>(stream), &enc_fail);
  if (enc_fail) return fail(VMLA_ERR_CUDA, "query_projection: tensor-map encoding failed");
  if (e != cudaSuccess) return cuda_fail(e, "query_projection launch");
  return VMLA_OK;
}

vmla_status vmla_output_projection(const uint16_t* o, const uint16_t* w_o, int32_t batch, int32_t n_tok,
                                   int32_t heads, int32_t d_model, uint16_t* y, void* stream) {
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(y))
    return fail(VMLA_ERR_INVALID_ARG, "output_projection: pointers must be non-null and 16-byte aligned");
  if (batch < 1 || n_tok < 1 || (int64_t)batch * n_tok > 0x7FFFFFFF)
    return fail(VMLA_ERR_INVALID_ARG, "output_projection: need batch, n_tok >= 1 and batch*n_tok < 2^31");
  if (heads < 1 || heads > 512) return fail(VMLA_ERR_INVALID_ARG, "output_projection: heads must be in [1, 512]");
  if (d_model < 128 || d_model > 65536 || d_model % 128 != 0)
    return fail(VMLA_ERR_UNSUPPORTED, "output_projection: d_model must be a multiple of 128 in [128, 65536]");
  if (((int64_t)batch * n_tok + 255) / 256 * ((d_model + 255) / 256) > 0x7FFFFFFF)
    return fail(VMLA_ERR_UNSUPPORTED, "output_projection: more than 2^31 - 1 output tiles");
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "output_projection: no CUDA device");
  bool enc_fail = false;
  cudaError_t e = vmla::launch_gemm_pair(o, w_o, nullptr, batch * n_tok, d_model, 0, heads * vmla::kDh, y,
                                         (int64_t)d_model, nullptr, 0, status, static_cast<cudaStream_t>(stream),
                                         &enc_fail);
  if (enc_fail) return fail(VMLA_ERR_CUDA, "output_projection: tensor-map encoding failed");
  if (e != cudaSuccess) return cuda_fail(e, "output_projection launch");
  return VMLA_OK;
}

vmla_status vmla_get_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "get_device_status: stream synchronize");
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "get_device_status: no CUDA device");
  int code = 0;
  e = cudaMemcpy(&code, status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "get_device_status: read status");
  if (code != 0) {
    const int zero = 0;
    e = cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "get_device_status: clear status");
    return fail(VMLA_ERR_TIMEOUT, "a kernel wait ran out of time (device code %d)", code);
  }
  return VMLA_OK;
}

vmla_status vmla_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll)
    return fail(VMLA_ERR_INVALID_ARG, "selftest_wait_timeout: limit_ns must be in [1e3, 1e10]");
  int* status = vmla::device_status_word();
  if (!status) return fail(VMLA_ERR_CUDA, "selftest_wait_timeout: no CUDA device");
  cudaError_t e = vmla::launch_selftest_wait_timeout(status, (uint64_t)limit_ns,
                                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest_wait_timeout launch");
  return VMLA_OK;
}

}  // extern "C"
