// Latent-cache append: c = x . W_DKV^T, k_r = RoPE3D(x . W_KR^T), 16-byte row writes.
//
// VideoMLA ("Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
// Diffusion", abstract and summary "Approach"): each cached token stores a
// head-shared content latent (d_c = 192 in the paper's model; the kernel is a
// template over d_c in {64, 128, 192, 256}) and a head-shared decoupled 3D-RoPE
// key (32).
//
// The arithmetic order is fixed so the result is reproducible bit for bit:
// every output is one fp32 accumulator updated for k = 0, 1, ..., d_model-1
// with fma(x_k, w_k, acc) -- bf16 x bf16 products are exact in fp32, so each step
// equals fl(acc + x_k w_k) -- then the rope pairs are rotated with separately
// rounded products and sums (__fmul_rn / __fadd_rn / __fsub_rn, no contraction),
// then rounded to bf16 (nearest even).  This is CUDA-core work: the tensor
// cores do not specify their accumulation order.
//
// Tiling: a CTA owns 32 tokens x all d_c + 32 outputs; each of its 8 warps owns
// 4 tokens, and lane l owns outputs l + 32 i, so the rope dims (the last 32
// outputs) sit one per lane and a pair (2p, 2p+1) lives in lanes (2p, 2p+1).
// Eight warps (two per scheduler) keep the FMA pipe fed through shared-memory
// latency; 32 tokens per CTA keep 480P's 4680-token chunk at one CTA per SM.
// Operands are staged per 64-wide k chunk in shared memory as fp32, double
// buffered: the global loads of chunk c+1 are issued into registers before the
// FMAs of chunk c, and land in the other buffer after them, so their latency
// hides behind the arithmetic.
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {

namespace {
constexpr int kKc = 64;          // k chunk
constexpr int kStride = kKc + 4; // fp32 row stride in shared memory (conflict-free float4 reads)

// A CTA owns 32 tokens x all d_c + 32 outputs.  Each warp owns 32 / kWarps
// tokens; lane l owns outputs l + 32 i.  Eight warps (two per scheduler, 4 tokens
// each) measured fastest for d_c >= 128; at d_c = 64 (three outputs per lane)
// four warps of 8 tokens reuse each loaded W value over more tokens and win.
template <int kDcT>
struct AppendCfg {
  static constexpr int kRow = kDcT + kDr;                    // cached scalars per token
  static constexpr int kWarps = kDcT == 64 ? 4 : 8;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kTok = 32;                            // tokens per CTA
  static constexpr int kTokPerWarp = kTok / kWarps;          // 8 or 4
  static constexpr int kOutPerLane = kRow / 32;              // 3, 5, 7, 9
  static constexpr int kBufFloats = (kRow + kTok) * kStride;
  static constexpr int kSmemBytes = 2 * kBufFloats * 4;
  static constexpr int kWVec = kRow * 8 / kThreads;          // 16-byte W vectors per thread per chunk
  static constexpr int kXVec = kTok * 8 / kThreads;          // 16-byte x vectors per thread per chunk
  static_assert(kRow % 32 == 0 && (kRow * 8) % kThreads == 0 && (kTok * 8) % kThreads == 0, "tiling");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// One 4-wide k step of a thread's kO outputs for its kT tokens.  x is stored
// rotated within each group of four (k+3, k, k+1, k+2), so the two operands of an
// FMA never sit in the same component of their vectors (fewer register-bank
// conflicts).  Every accumulator takes k, k+1, k+2, k+3 in turn (its sequential
// order), and consecutive FMAs belong to different accumulators.
template <int kT, int kO>
__device__ __forceinline__ void fma_step(float (&acc)[kT][kO], const float* ws, const float* xs, int lane,
                                         int tok_row0, int kk) {
  float4 wv[kO];
#pragma unroll
  for (int i = 0; i < kO; ++i) wv[i] = *reinterpret_cast<const float4*>(ws + (lane + 32 * i) * kStride + kk);
  float4 xv[kT];
#pragma unroll
  for (int t = 0; t < kT; ++t) xv[t] = *reinterpret_cast<const float4*>(xs + (tok_row0 + t) * kStride + kk);
#pragma unroll
  for (int t = 0; t < kT; ++t)
#pragma unroll
    for (int i = 0; i < kO; ++i) acc[t][i] = fmaf(xv[t].y, wv[i].x, acc[t][i]);  // k
#pragma unroll
  for (int t = 0; t < kT; ++t)
#pragma unroll
    for (int i = 0; i < kO; ++i) acc[t][i] = fmaf(xv[t].z, wv[i].y, acc[t][i]);  // k + 1
#pragma unroll
  for (int t = 0; t < kT; ++t)
#pragma unroll
    for (int i = 0; i < kO; ++i) acc[t][i] = fmaf(xv[t].w, wv[i].z, acc[t][i]);  // k + 2
#pragma unroll
  for (int t = 0; t < kT; ++t)
#pragma unroll
    for (int i = 0; i < kO; ++i) acc[t][i] = fmaf(xv[t].x, wv[i].w, acc[t][i]);  // k + 3
}

struct AppendParams {
  const uint16_t* x;
  const uint16_t* w_dkv;
  const uint16_t* w_kr;
  uint16_t* cache;
  int64_t cap;
  int64_t slot0;
  int n_tok;
  int d_model;
  int grid_h;
  int grid_w;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float4& lo, float4& hi) {
  lo = make_float4(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y));
  hi = make_float4(bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w));
}

template <int kDcT>
__global__ void __launch_bounds__(AppendCfg<kDcT>::kThreads, 1)
    k_cache_append(const __grid_constant__ AppendParams p, const __grid_constant__ RopeTable tab) {
  using A = AppendCfg<kDcT>;
  constexpr int kDrow = A::kRow, kTok = A::kTok, kTokPerWarp = A::kTokPerWarp, kOutPerLane = A::kOutPerLane;
  constexpr int kBufFloats = A::kBufFloats, kWVec = A::kWVec, kXVec = A::kXVec, kThreads = A::kThreads;
  extern __shared__ __align__(16) float smem_f[];
  const int b = blockIdx.y;
  const int tok0 = blockIdx.x * kTok;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint16_t* xb = p.x + (int64_t)b * p.n_tok * p.d_model;

  float acc[kTokPerWarp][kOutPerLane];
#pragma unroll
  for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
    for (int i = 0; i < kOutPerLane; ++i) acc[t][i] = 0.0f;

  // Register staging of one k chunk: vector v = threadIdx.x + kThreads * n.
  uint4 wreg[kWVec], xreg[kXVec];
  auto load_chunk = [&](int k0) {
#pragma unroll
    for (int n = 0; n < kWVec; ++n) {
      const int v = threadIdx.x + kThreads * n;
      const int row = v >> 3, kk = (v & 7) * 8;
      const uint16_t* src = row < kDcT ? p.w_dkv + (int64_t)row * p.d_model
                                       : p.w_kr + (int64_t)(row - kDcT) * p.d_model;
      wreg[n] = __ldg(reinterpret_cast<const uint4*>(src + k0 + kk));
    }
#pragma unroll
    for (int n = 0; n < kXVec; ++n) {
      const int v = threadIdx.x + kThreads * n;
      const int t = v >> 3, kk = (v & 7) * 8;
      xreg[n] = tok0 + t < p.n_tok
                    ? __ldg(reinterpret_cast<const uint4*>(xb + (int64_t)(tok0 + t) * p.d_model + k0 + kk))
                    : make_uint4(0, 0, 0, 0);
    }
  };
  auto store_chunk = [&](float* buf) {
    float* ws = buf;
    float* xs = buf + kDrow * kStride;
#pragma unroll
    for (int n = 0; n < kWVec; ++n) {
      const int v = threadIdx.x + kThreads * n;
      const int row = v >> 3, kk = (v & 7) * 8;
      float4 lo, hi;
      bf16x8_to_f32(wreg[n], lo, hi);
      *reinterpret_cast<float4*>(ws + row * kStride + kk) = lo;
      *reinterpret_cast<float4*>(ws + row * kStride + kk + 4) = hi;
    }
#pragma unroll
    for (int n = 0; n < kXVec; ++n) {
      const int v = threadIdx.x + kThreads * n;
      const int t = v >> 3, kk = (v & 7) * 8;
      float4 lo, hi;
      bf16x8_to_f32(xreg[n], lo, hi);
      *reinterpret_cast<float4*>(xs + t * kStride + kk) = make_float4(lo.w, lo.x, lo.y, lo.z);
      *reinterpret_cast<float4*>(xs + t * kStride + kk + 4) = make_float4(hi.w, hi.x, hi.y, hi.z);
    }
  };

  const int n_chunks = p.d_model / kKc;
  load_chunk(0);
  store_chunk(smem_f);
  __syncthreads();
  for (int c = 0; c < n_chunks; ++c) {
    const float* ws = smem_f + (c & 1) * kBufFloats;
    const float* xs = ws + kDrow * kStride;
    if (c + 1 < n_chunks) load_chunk((c + 1) * kKc);
#pragma unroll 2
    for (int kk = 0; kk < kKc; kk += 4) fma_step(acc, ws, xs, lane, warp * kTokPerWarp, kk);
    if (c + 1 < n_chunks) store_chunk(smem_f + ((c + 1) & 1) * kBufFloats);
    __syncthreads();
  }

  // 3D rotary embedding of the rope dims: output d_c + lane is the lane's last output.
  constexpr int kRope = kOutPerLane - 1;
  {
    const int pair = lane >> 1;
    const bool even = (lane & 1) == 0;
    const int per_frame = p.grid_h * p.grid_w;
#pragma unroll
    for (int t = 0; t < kTokPerWarp; ++t) {
      const int tok = tok0 + warp * kTokPerWarp + t;
      const float v = acc[t][kRope];
      const float other = __shfl_xor_sync(0xffffffffu, v, 1);
      if (tok < p.n_tok) {
        const int f = tok / per_frame;
        const int rem = tok - f * per_frame;
        const int row = rem / p.grid_w;
        const int col = rem - row * p.grid_w;
        float2 cs;
        if (pair < kPairsT) cs = tab.t[f][pair];
        else if (pair < kPairsT + kPairsH) cs = tab.h[row][pair - kPairsT];
        else cs = tab.w[col][pair - kPairsT - kPairsH];
        const float a = even ? v : other;
        const float bb = even ? other : v;
        acc[t][kRope] = even ? __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(bb, cs.y))
                             : __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(bb, cs.x));
      }
    }
  }

  // Stage the kTok x (d_c + 32) bf16 rows in shared memory, then write 16-byte vectors.
  __syncthreads();
  __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(smem_f);
#pragma unroll
  for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
    for (int i = 0; i < kOutPerLane; ++i)
      os[(warp * kTokPerWarp + t) * kDrow + lane + 32 * i] = __float2bfloat16_rn(acc[t][i]);
  __syncthreads();
  constexpr int kVecPerRow = kDrow * 2 / 16;
  for (int v = threadIdx.x; v < kTok * kVecPerRow; v += kThreads) {
    const int t = v / kVecPerRow, c = v - t * kVecPerRow;
    const int tok = tok0 + t;
    if (tok < p.n_tok) {
      const int64_t slot = (p.slot0 + tok) % p.cap;
      uint4 val = *reinterpret_cast<const uint4*>(os + t * kDrow + c * 8);
      *reinterpret_cast<uint4*>(p.cache + ((int64_t)b * p.cap + slot) * kDrow + c * 8) = val;
    }
  }
}

template <int kDcT>
cudaError_t launch_cache_append_t(const AppendParams& p, int batch, int64_t t0, cudaStream_t stream) {
  using A = AppendCfg<kDcT>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_cache_append<kDcT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         A::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  static thread_local RopeTable tab;
  const int per_frame = p.grid_h * p.grid_w;
  build_rope_table(&tab, t0, (p.n_tok + per_frame - 1) / per_frame, p.grid_h, p.grid_w);
  dim3 grid((p.n_tok + A::kTok - 1) / A::kTok, batch);
  k_cache_append<kDcT><<<grid, A::kThreads, A::kSmemBytes, stream>>>(p, tab);
  return cudaGetLastError();
}
}  // namespace

// d_c in {64, 128, 192, 256}; the caller has validated it.
cudaError_t launch_cache_append(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                                int batch, int n_tok, int d_model, int d_c, uint16_t* cache, int64_t cap,
                                int64_t slot0, int64_t t0, int grid_h, int grid_w,
                                cudaStream_t stream) {
  AppendParams p{x, w_dkv, w_kr, cache, cap, slot0, n_tok, d_model, grid_h, grid_w};
  switch (d_c) {
    case 64: return launch_cache_append_t<64>(p, batch, t0, stream);
    case 128: return launch_cache_append_t<128>(p, batch, t0, stream);
    case 192: return launch_cache_append_t<192>(p, batch, t0, stream);
    case 256: return launch_cache_append_t<256>(p, batch, t0, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vmla
