// Latent-cache append: c = x . W_DKV^T, k_r = RoPE3D(x . W_KR^T), 16-byte row writes.
//
// VideoMLA ("Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
// Diffusion", abstract and summary "Approach"): each cached token stores a
// head-shared content latent (d_c = 192 in the paper's model; the kernels are
// templates over d_c in {64, 128, 192, 256}) and a head-shared decoupled 3D-RoPE
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
// What bounds it.  A CTA owns 32 tokens x all d_c + 32 outputs, and 480P's
// 4680-token chunk is one such tile per SM.  Shared memory delivers 32 four-byte
// words per clock whatever the access width or broadcast, so the operand words a
// thread reads per FMA decide the speed once the FMAs are spread over enough
// threads to keep the schedulers busy.  Hence:
//  - W stays bf16 in shared memory (half the words of fp32) and is widened in
//    registers (exact: a bf16 is the top half of an fp32), one instruction per
//    W value;
//  - the FMAs of two outputs of a token are issued as one fma.rn.f32x2 (two
//    separately rounded fp32 FMAs, the same bits as two fmaf), which frees the
//    issue slots the widening costs;
//  - x is widened to fp32 once per CTA when it is staged, except in the wide
//    layout at d_c >= 192, where it too stays bf16 and is widened per use (its
//    loads then take half the shared-memory wavefronts).
// Two thread layouts share this scheme:
//  - wide (8 warps, two per scheduler): warp w owns tokens 4w .. 4w+3, lane l
//    owns outputs l + 32 i.  Used when each SM holds one tile.
//  - tall (4 warps): lanes form 4 token groups x 8 output groups and a thread
//    holds 8 tokens x (d_c + 32) / 32 outputs, half the operand words per FMA of
//    the wide form.  With one warp per scheduler it stalls more, so it only wins
//    where two tiles share an SM (more tiles than SMs, d_c <= 192).
//  - slice (8 warps): for appends too small to fill the SMs, a CTA computes one
//    64-output slice (or the rope slice) of a tile, so the tile's slices run on
//    separate SMs.
//
// Operands per 64-wide k chunk: W (d_c + 32 rows of bf16) is copied by
// cp.async into a 3-stage ring; x (32 rows) is loaded one chunk ahead into
// registers and stored (widened, or as bf16) into a double buffer.  The k steps
// of a chunk are software pipelined: the loads of step s + 1 are spread over the
// FMAs of step s.
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {

namespace {
constexpr int kKc = 64;             // k chunk
constexpr int kTok = 32;            // tokens per CTA
constexpr int kXStride = kKc + 8;   // fp32 x row stride in shared memory (72 words)
constexpr int kWStride = kKc + 8;   // bf16 W row stride in shared memory (144 bytes)
constexpr int kWStages = 3;

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

// Shared-memory plan and staging shares of a layout with kThreads threads; with
// kXRaw, x rows stay bf16 (kWStride elements per row).
template <int kDcT, int kThreads, bool kXRaw = false>
struct Stage {
  static constexpr int kRow = kDcT + kDr;                    // cached scalars per token
  static constexpr int kWStageBytes = kRow * kWStride * 2;
  static constexpr int kXBufFloats = kXRaw ? kTok * kWStride / 2 : kTok * kXStride;
  static constexpr int kSmemBytes = kWStages * kWStageBytes + 2 * kXBufFloats * 4;
  static constexpr int kWCopies = kRow * (kKc / 8) / kThreads;  // 16-byte W copies per thread per chunk
  static constexpr int kXVec = kTok * (kKc / 8) / kThreads;     // 16-byte x loads per thread per chunk
  static_assert(kRow % 32 == 0, "rows");
  static_assert((kRow * (kKc / 8)) % kThreads == 0 && (kTok * (kKc / 8)) % kThreads == 0, "staging");
  static_assert(kTok * kRow * 2 <= kSmemBytes, "output staging");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kN>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kN) : "memory"); }

__device__ __forceinline__ uint32_t u4comp(const uint4& v, int e) {
  return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}
__device__ __forceinline__ float f4comp(const float4& v, int e) {
  return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}
// k value e of a bf16 pair word (e even: the low half).
__device__ __forceinline__ float widen(uint32_t word, int e) {
  return (e & 1) ? bf16hi_to_f32(word) : bf16lo_to_f32(word);
}

// The chunk pipeline shared by both layouts: W ring by cp.async, x staged
// through registers, one __syncthreads per chunk.  `compute(xs, ws)` runs the
// FMAs of one chunk.
template <int kDcT, int kThreads, bool kXRaw, class Compute>
__device__ __forceinline__ void run_chunks(const AppendParams& p, uint8_t* smem_raw, int b, int tok0,
                                           Compute&& compute) {
  using S = Stage<kDcT, kThreads, kXRaw>;
  uint16_t* wring = reinterpret_cast<uint16_t*>(smem_raw);
  float* xbuf = reinterpret_cast<float*>(smem_raw + kWStages * S::kWStageBytes);
  const uint32_t wring_s = static_cast<uint32_t>(__cvta_generic_to_shared(wring));
  const uint16_t* xb = p.x + (int64_t)b * p.n_tok * p.d_model;
  const int n_chunks = p.d_model / kKc;

  // W chunk c -> ring stage c % kWStages: copy v = threadIdx.x + kThreads * n is
  // row v / 8, bytes 16 (v % 8) of the row's 128.
  auto issue_w = [&](int c) {
    if (c < n_chunks) {
      const uint32_t dst0 = wring_s + (c % kWStages) * S::kWStageBytes;
#pragma unroll
      for (int n = 0; n < S::kWCopies; ++n) {
        const int v = threadIdx.x + kThreads * n;
        const int row = v >> 3, kk = (v & 7) * 8;
        const uint16_t* src = row < kDcT ? p.w_dkv + (int64_t)row * p.d_model
                                         : p.w_kr + (int64_t)(row - kDcT) * p.d_model;
        cp_async16(dst0 + (row * kWStride + kk) * 2, src + c * kKc + kk);
      }
    }
    cp_async_commit();  // one group per chunk index, empty past the end
  };
  // x chunk: vector v = threadIdx.x + kThreads * n is token v / 8, k (v % 8) * 8.
  uint4 xreg[S::kXVec];
  auto load_x = [&](int c) {
#pragma unroll
    for (int n = 0; n < S::kXVec; ++n) {
      const int v = threadIdx.x + kThreads * n;
      const int t = v >> 3, kk = (v & 7) * 8;
      xreg[n] = tok0 + t < p.n_tok
                    ? __ldg(reinterpret_cast<const uint4*>(xb + (int64_t)(tok0 + t) * p.d_model + c * kKc + kk))
                    : make_uint4(0, 0, 0, 0);
    }
  };
  auto store_x = [&](float* xs) {
#pragma unroll
    for (int n = 0; n < S::kXVec; ++n) {
      const int v = threadIdx.x + kThreads * n;
      const int t = v >> 3, kk = (v & 7) * 8;
      const uint4 u = xreg[n];
      if constexpr (kXRaw) {
        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(xs) + t * kWStride + kk) = u;
        continue;
      }
      *reinterpret_cast<float4*>(xs + t * kXStride + kk) =
          make_float4(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y), bf16hi_to_f32(u.y));
      *reinterpret_cast<float4*>(xs + t * kXStride + kk + 4) =
          make_float4(bf16lo_to_f32(u.z), bf16hi_to_f32(u.z), bf16lo_to_f32(u.w), bf16hi_to_f32(u.w));
    }
  };

#pragma unroll
  for (int c = 0; c < kWStages - 1; ++c) issue_w(c);
  load_x(0);
  store_x(xbuf);
  if (n_chunks > 1) load_x(1);
  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<kWStages - 2>();  // this thread's copies of chunk c have landed
    __syncthreads();                // everyone's have, and chunk c - 1 is consumed
    issue_w(c + kWStages - 1);      // into the stage chunk c - 1 used
    if (c + 1 < n_chunks) {
      store_x(xbuf + ((c + 1) & 1) * S::kXBufFloats);
      if (c + 2 < n_chunks) load_x(c + 2);
    }
    compute(xbuf + (c & 1) * S::kXBufFloats, wring + (c % kWStages) * (S::kWStageBytes / 2));
  }
  cp_async_wait<0>();
}

// Rotates the rope value v of token `tok` (pair `pair`; `other` is the partner
// lane's value, `even` whether this lane holds the pair's first dim).
__device__ __forceinline__ float rope_rotate(const AppendParams& p, const RopeTable& tab, int tok, int pair,
                                             bool even, float v, float other) {
  const int per_frame = p.grid_h * p.grid_w;
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
  return even ? __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(bb, cs.y))
              : __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(bb, cs.x));
}

// Writes the CTA's staged bf16 rows (kTok x kRow in shared memory) to their ring
// slots as 16-byte vectors.
template <int kRow, int kThreads>
__device__ __forceinline__ void write_rows(const AppendParams& p, const __nv_bfloat16* os, int b, int tok0) {
  constexpr int kVecPerRow = kRow * 2 / 16;
  for (int v = threadIdx.x; v < kTok * kVecPerRow; v += kThreads) {
    const int t = v / kVecPerRow, c = v - t * kVecPerRow;
    const int tok = tok0 + t;
    if (tok < p.n_tok) {
      const int64_t slot = (p.slot0 + tok) % p.cap;
      const uint4 val = *reinterpret_cast<const uint4*>(os + t * kRow + c * 8);
      *reinterpret_cast<uint4*>(p.cache + ((int64_t)b * p.cap + slot) * kRow + c * 8) = val;
    }
  }
}

// ---- wide layout ------------------------------------------------------------
//
// Warp w owns tokens 4w .. 4w+3; lane l owns outputs l + 32 i, i < kN: kP content
// pairs (l + 64 q, l + 64 q + 32) and the rope dim d_c + l.  k steps are 8 wide:
// one 16-byte load per W row (8 bf16) and two per x row.  For a W load the 8
// rows of a quarter-warp start 144 bytes apart (distinct 16-byte bank groups);
// an x load is one address for the whole warp.
template <int kDcT>
struct Wide {
  static constexpr int kRow = kDcT + kDr;
  static constexpr int kN = kRow / 32;      // outputs per lane: 3, 5, 7, 9
  static constexpr int kP = (kN - 1) / 2;   // content pairs per lane
  static constexpr int kWarps = 8;
  static constexpr int kT = kTok / kWarps;  // tokens per warp
  static constexpr int kThreads = 32 * kWarps;
  // x stays bf16 in shared memory (widened per use, like W) at d_c >= 192, where
  // the halved x wavefronts pay for the widening; at d_c = 64 and 128 it is
  // staged as fp32.
  static constexpr bool kXRaw = kDcT >= 192;
  using S = Stage<kDcT, kThreads, kXRaw>;
  static_assert(kDcT == 64 * kP, "kP content pairs + one rope dim per lane");

  // x[t][h]: fp32 k + 4h .. k + 4h + 3 of token row tok_row0 + t, or (kXRaw)
  // x[t][0] = 8 bf16 of that row.
  struct Frag {
    uint4 w[kN];
    float4 x[kT][kXRaw ? 1 : 2];
  };
  static constexpr int kXLoads = kXRaw ? 1 : 2;   // x loads per token per step
  __device__ static __forceinline__ float4 load_x(const float* xs, int row, int kk, int h) {
    if constexpr (kXRaw) {
      return *reinterpret_cast<const float4*>(reinterpret_cast<const uint16_t*>(xs) + row * kWStride + kk);
    } else {
      return *reinterpret_cast<const float4*>(xs + row * kXStride + kk + 4 * h);
    }
  }
  // fp32 value of x at k offset e (0..7) of the step.
  __device__ static __forceinline__ float x_at(const float4 (&x)[kXRaw ? 1 : 2], int e) {
    if constexpr (kXRaw) {
      const float4 v = x[0];
      return widen(__float_as_uint(f4comp(v, e >> 1)), e);
    } else {
      return f4comp(x[e >> 2], e & 3);
    }
  }

  __device__ static __forceinline__ void load(Frag& f, const float* xs, const uint16_t* ws, int lane,
                                              int tok_row0, int kk) {
#pragma unroll
    for (int i = 0; i < kN; ++i) f.w[i] = *reinterpret_cast<const uint4*>(ws + (lane + 32 * i) * kWStride + kk);
#pragma unroll
    for (int t = 0; t < kT; ++t)
#pragma unroll
      for (int h = 0; h < kXLoads; ++h) f.x[t][h] = load_x(xs, tok_row0 + t, kk, h);
  }

  // One 8-wide k step on `cur`; the loads of the next step (k offset kk_next)
  // into `nxt` are spread over it, about two per k.  Every accumulator takes
  // k, k+1, ..., k+7 in turn (its sequential order).
  __device__ static __forceinline__ void step(float2 (&acc2)[kT][kP], float (&acc1)[kT], const Frag& cur,
                                              Frag& nxt, const float* xs, const uint16_t* ws, int lane,
                                              int tok_row0, int kk_next) {
    constexpr int kLoads = kN + kXLoads * kT;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
      for (int n = (kLoads * e) / 8; n < (kLoads * (e + 1)) / 8; ++n) {
        if (n < kN) {
          nxt.w[n] = *reinterpret_cast<const uint4*>(ws + (lane + 32 * n) * kWStride + kk_next);
        } else {
          const int t = (n - kN) / kXLoads, h = (n - kN) % kXLoads;
          nxt.x[t][h] = load_x(xs, tok_row0 + t, kk_next, h);
        }
      }
      float wf[kN];
#pragma unroll
      for (int i = 0; i < kN; ++i) wf[i] = widen(u4comp(cur.w[i], e >> 1), e);
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const float xv = x_at(cur.x[t], e);
        const float2 xx = make_float2(xv, xv);
#pragma unroll
        for (int q = 0; q < kP; ++q)
          acc2[t][q] = __ffma2_rn(xx, make_float2(wf[2 * q], wf[2 * q + 1]), acc2[t][q]);
        acc1[t] = fmaf(xv, wf[kN - 1], acc1[t]);
      }
    }
  }
};

template <int kDcT>
__global__ void __launch_bounds__(Wide<kDcT>::kThreads, 1)
    k_cache_append_wide(const __grid_constant__ AppendParams p, const __grid_constant__ RopeTable tab) {
  using L = Wide<kDcT>;
  constexpr int kT = L::kT, kP = L::kP, kRow = L::kRow;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int b = blockIdx.y;
  const int tok0 = blockIdx.x * kTok;
  const int lane = threadIdx.x & 31;
  const int tok_row0 = (threadIdx.x >> 5) * kT;   // this warp's first token row (within the CTA)

  float2 acc2[kT][kP];   // outputs (lane + 64 q, lane + 64 q + 32)
  float acc1[kT];        // output d_c + lane (rope)
#pragma unroll
  for (int t = 0; t < kT; ++t) {
#pragma unroll
    for (int q = 0; q < kP; ++q) acc2[t][q] = make_float2(0.0f, 0.0f);
    acc1[t] = 0.0f;
  }

  run_chunks<kDcT, L::kThreads, L::kXRaw>(p, smem_raw, b, tok0, [&](const float* xs, const uint16_t* ws) {
    // Steps in pairs (f0 -> f1 -> f0); the last step's prefetch reads the row
    // padding at k offset 64 (in bounds, never used).
    typename L::Frag f0, f1;
    L::load(f0, xs, ws, lane, tok_row0, 0);
#pragma unroll 2
    for (int kk = 0; kk < kKc; kk += 16) {
      L::step(acc2, acc1, f0, f1, xs, ws, lane, tok_row0, kk + 8);
      L::step(acc2, acc1, f1, f0, xs, ws, lane, tok_row0, kk + 16);
    }
  });

  // Rope: output d_c + lane is acc1; a pair (2p, 2p+1) sits in lanes (2p, 2p+1).
#pragma unroll
  for (int t = 0; t < kT; ++t) {
    const int tok = tok0 + tok_row0 + t;
    const float other = __shfl_xor_sync(0xffffffffu, acc1[t], 1);
    if (tok < p.n_tok) acc1[t] = rope_rotate(p, tab, tok, lane >> 1, (lane & 1) == 0, acc1[t], other);
  }

  __syncthreads();
  __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(smem_raw);
#pragma unroll
  for (int t = 0; t < kT; ++t) {
    __nv_bfloat16* orow = os + (tok_row0 + t) * kRow;
#pragma unroll
    for (int q = 0; q < kP; ++q) {
      orow[lane + 64 * q] = __float2bfloat16_rn(acc2[t][q].x);
      orow[lane + 64 * q + 32] = __float2bfloat16_rn(acc2[t][q].y);
    }
    orow[kDcT + lane] = __float2bfloat16_rn(acc1[t]);
  }
  __syncthreads();
  write_rows<kRow, L::kThreads>(p, os, b, tok0);
}

// ---- tall layout ------------------------------------------------------------
//
// Lane l = 8 g + j: token group g (0..3), output group j (0..7); warp q owns
// output quarter q.  A thread holds tokens g + 4 t (t < 8) and outputs
// q * 8 kN + j + 8 m (m < kN): pairs (m = 2r, 2r + 1) and a single m = kN - 1.
// k steps are 4 wide: one 8-byte load per W row (4 bf16), one 16-byte load per
// x row.  For a W load the 8 rows j of a half-warp start 144 bytes apart
// (distinct bank pairs); an x load is one address per quarter-warp.
template <int kDcT>
struct Tall {
  static constexpr int kRow = kDcT + kDr;
  static constexpr int kN = kRow / 32;      // outputs per thread: 3, 5, 7, 9
  static constexpr int kP = kN / 2;         // output pairs per thread
  static constexpr int kT = 8;              // tokens per thread
  static constexpr int kThreads = 128;
  using S = Stage<kDcT, kThreads>;
  static_assert(kN % 2 == 1, "kP pairs + one single output per thread");

  struct Frag {
    float4 x[kT];
    uint2 w[kN];
  };

  __device__ static __forceinline__ void load(Frag& f, const float* xs, const uint16_t* ws, int x_row0,
                                              int w_row0, int kk) {
#pragma unroll
    for (int m = 0; m < kN; ++m) f.w[m] = *reinterpret_cast<const uint2*>(ws + (w_row0 + 8 * m) * kWStride + kk);
#pragma unroll
    for (int t = 0; t < kT; ++t) f.x[t] = *reinterpret_cast<const float4*>(xs + (x_row0 + 4 * t) * kXStride + kk);
  }

  // One 4-wide k step on `cur`; the loads of the next step (k offset kk_next)
  // into `nxt` are spread over it, a quarter before each k's FMAs.  Every
  // accumulator takes k, k+1, k+2, k+3 in turn (its sequential order).
  __device__ static __forceinline__ void step(float2 (&acc2)[kT][kP], float (&acc1)[kT], const Frag& cur,
                                              Frag& nxt, const float* xs, const uint16_t* ws, int x_row0,
                                              int w_row0, int kk_next) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
      for (int m = e; m < kN; m += 4)
        nxt.w[m] = *reinterpret_cast<const uint2*>(ws + (w_row0 + 8 * m) * kWStride + kk_next);
#pragma unroll
      for (int t = e; t < kT; t += 4)
        nxt.x[t] = *reinterpret_cast<const float4*>(xs + (x_row0 + 4 * t) * kXStride + kk_next);
      float wf[kN];
#pragma unroll
      for (int m = 0; m < kN; ++m) wf[m] = widen((e < 2) ? cur.w[m].x : cur.w[m].y, e);
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const float xv = f4comp(cur.x[t], e);
        const float2 xx = make_float2(xv, xv);
#pragma unroll
        for (int r = 0; r < kP; ++r)
          acc2[t][r] = __ffma2_rn(xx, make_float2(wf[2 * r], wf[2 * r + 1]), acc2[t][r]);
        acc1[t] = fmaf(xv, wf[kN - 1], acc1[t]);
      }
    }
  }
};

template <int kDcT>
__global__ void __launch_bounds__(Tall<kDcT>::kThreads, 1)
    k_cache_append_tall(const __grid_constant__ AppendParams p, const __grid_constant__ RopeTable tab) {
  using L = Tall<kDcT>;
  constexpr int kT = L::kT, kN = L::kN, kP = L::kP, kRow = L::kRow;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int b = blockIdx.y;
  const int tok0 = blockIdx.x * kTok;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int j = lane & 7;
  const int x_row0 = lane >> 3;               // first token row of this thread (within the CTA)
  const int w_row0 = warp * 8 * kN + j;       // first output row of this thread

  // Output m of token t: acc2[t][m / 2].x / .y for m < kN - 1, acc1[t] for m = kN - 1.
  float2 acc2[kT][kP];
  float acc1[kT];
#pragma unroll
  for (int t = 0; t < kT; ++t) {
#pragma unroll
    for (int r = 0; r < kP; ++r) acc2[t][r] = make_float2(0.0f, 0.0f);
    acc1[t] = 0.0f;
  }
  auto acc = [&](int t, int m) -> float& {
    return m == kN - 1 ? acc1[t] : ((m & 1) ? acc2[t][m >> 1].y : acc2[t][m >> 1].x);
  };

  run_chunks<kDcT, L::kThreads, false>(p, smem_raw, b, tok0, [&](const float* xs, const uint16_t* ws) {
    // Steps in pairs (f0 -> f1 -> f0); the last step's prefetch reads the row
    // padding at k offset 64 (in bounds, never used).
    typename L::Frag f0, f1;
    L::load(f0, xs, ws, x_row0, w_row0, 0);
#pragma unroll 2
    for (int kk = 0; kk < kKc; kk += 8) {
      L::step(acc2, acc1, f0, f1, xs, ws, x_row0, w_row0, kk + 4);
      L::step(acc2, acc1, f1, f0, xs, ws, x_row0, w_row0, kk + 8);
    }
  });

  // Rope: whether output w_row0 + 8 m is a rope dim is the same for the whole
  // warp (d_c is a multiple of 8), and a pair (2p, 2p+1) sits in lanes j, j ^ 1.
#pragma unroll
  for (int m = 0; m < kN; ++m) {
    const int o = w_row0 + 8 * m;
    if (o - j < kDcT) continue;
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      const int tok = tok0 + x_row0 + 4 * t;
      const float other = __shfl_xor_sync(0xffffffffu, acc(t, m), 1);
      if (tok < p.n_tok) acc(t, m) = rope_rotate(p, tab, tok, (o - kDcT) >> 1, (j & 1) == 0, acc(t, m), other);
    }
  }

  __syncthreads();
  __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(smem_raw);
#pragma unroll
  for (int t = 0; t < kT; ++t)
#pragma unroll
    for (int m = 0; m < kN; ++m) os[(x_row0 + 4 * t) * kRow + w_row0 + 8 * m] = __float2bfloat16_rn(acc(t, m));
  __syncthreads();
  write_rows<kRow, L::kThreads>(p, os, b, tok0);
}

// ---- slice layout -----------------------------------------------------------
//
// For appends too small to fill the SMs: the d_c + 32 outputs are cut into d_c/64
// content slices of 64 rows and the 32-row rope slice, and a CTA computes one
// slice for 32 tokens (grid z = slice), so a chunk of T tiles runs as
// T (d_c/64 + 1) CTAs.  8 warps of 4 tokens; in a content slice lane l owns rows
// s0 + l and s0 + 32 + l (one paired FMA), in the rope slice row d_c + l.  Both
// W and x stay bf16 in shared memory and arrive by cp.async through an 8-stage
// ring (a stage is only 64 W rows + 32 x rows).  A 3-stage ring timed the same,
// so the depth is not what hides the loads; at 8 stages a CTA takes 110.6 KB, and
// two of them still fit on an SM, which the launcher's two-per-SM rule checks
// with the occupancy API.  Same arithmetic order as the other layouts.
template <int kDcT>
struct Slice {
  static constexpr int kRow = kDcT + kDr;
  static constexpr int kParts = kDcT / 64 + 1;   // content slices + the rope slice
  static constexpr int kWRows = 64;
  static constexpr int kWarps = 8;
  static constexpr int kT = kTok / kWarps;       // tokens per warp
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kStages = 8;
  static constexpr int kStageBytes = (kWRows + kTok) * kWStride * 2;   // W rows, then x rows
  static constexpr int kSmemBytes = kStages * kStageBytes;
  static constexpr int kCopies = (kWRows + kTok) * (kKc / 8) / kThreads;  // 16-byte copies per thread per chunk
  static_assert(((kWRows + kTok) * (kKc / 8)) % kThreads == 0, "staging");
  static_assert(kTok * kWRows * 2 <= kSmemBytes && kSmemBytes <= 232448, "shared memory");
};

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

// One CTA of the slice layout; kRope: the rope slice (rows d_c .. d_c + 31).
template <int kDcT, bool kRope>
__device__ __forceinline__ void slice_body(const AppendParams& p, const RopeTable& tab, uint8_t* smem_raw) {
  using L = Slice<kDcT>;
  constexpr int kT = L::kT, kRow = L::kRow, kStages = L::kStages;
  constexpr bool rope = kRope;
  const uint32_t ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const int b = blockIdx.y;
  const int tok0 = blockIdx.x * kTok;
  const int part = blockIdx.z;
  const int s0 = part * 64;                       // first output row of the slice
  constexpr int n_rows = kRope ? kDr : 64;
  const int lane = threadIdx.x & 31;
  const int tok_row0 = (threadIdx.x >> 5) * kT;
  const uint16_t* xb = p.x + (int64_t)b * p.n_tok * p.d_model;
  const int n_chunks = p.d_model / kKc;

  // Chunk c -> stage c % kStages: copy v = threadIdx.x + kThreads n is row v / 8
  // (W rows first, then the 32 x rows), bytes 16 (v % 8) of the row's 128.
  auto issue = [&](int c) {
    if (c < n_chunks) {
      const uint32_t dst0 = ring_s + (c % kStages) * L::kStageBytes;
#pragma unroll
      for (int n = 0; n < L::kCopies; ++n) {
        const int v = threadIdx.x + L::kThreads * n;
        const int row = v >> 3, kk = (v & 7) * 8;
        const uint32_t dst = dst0 + (row * kWStride + kk) * 2;
        if (row < L::kWRows) {
          if (row >= n_rows) continue;
          const int grow = s0 + row;
          const uint16_t* src = grow < kDcT ? p.w_dkv + (int64_t)grow * p.d_model
                                            : p.w_kr + (int64_t)(grow - kDcT) * p.d_model;
          cp_async16(dst, src + c * kKc + kk);
        } else {
          const int t = row - L::kWRows;
          const bool valid = tok0 + t < p.n_tok;
          cp_async16_zfill(dst, xb + (int64_t)(valid ? tok0 + t : 0) * p.d_model + c * kKc + kk, valid);
        }
      }
    }
    cp_async_commit();  // one group per chunk index, empty past the end
  };

  float2 acc[kT];   // content: rows (s0 + lane, s0 + 32 + lane); rope: .x is row d_c + lane
#pragma unroll
  for (int t = 0; t < kT; ++t) acc[t] = make_float2(0.0f, 0.0f);

#pragma unroll
  for (int c = 0; c < kStages - 1; ++c) issue(c);
  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<kStages - 2>();  // this thread's copies of chunk c have landed
    __syncthreads();                // everyone's have, and chunk c - 1 is consumed
    issue(c + kStages - 1);         // into the stage chunk c - 1 used
    const uint16_t* ws = reinterpret_cast<const uint16_t*>(smem_raw + (c % kStages) * L::kStageBytes);
    const uint16_t* xr = ws + L::kWRows * kWStride;
#pragma unroll 2
    for (int kk = 0; kk < kKc; kk += 8) {
      const uint4 w0 = *reinterpret_cast<const uint4*>(ws + lane * kWStride + kk);
      const uint4 w1 = rope ? w0 : *reinterpret_cast<const uint4*>(ws + (32 + lane) * kWStride + kk);
      uint4 xq[kT];
#pragma unroll
      for (int t = 0; t < kT; ++t) xq[t] = *reinterpret_cast<const uint4*>(xr + (tok_row0 + t) * kWStride + kk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float wa = widen(u4comp(w0, e >> 1), e);
        const float wb = widen(u4comp(w1, e >> 1), e);
#pragma unroll
        for (int t = 0; t < kT; ++t) {
          const float xv = widen(u4comp(xq[t], e >> 1), e);
          if constexpr (kRope) acc[t].x = fmaf(xv, wa, acc[t].x);
          else acc[t] = __ffma2_rn(make_float2(xv, xv), make_float2(wa, wb), acc[t]);
        }
      }
    }
  }
  cp_async_wait<0>();

  if constexpr (kRope) {  // a pair (2p, 2p+1) of rope dims sits in lanes (2p, 2p+1)
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      const int tok = tok0 + tok_row0 + t;
      const float other = __shfl_xor_sync(0xffffffffu, acc[t].x, 1);
      if (tok < p.n_tok) acc[t].x = rope_rotate(p, tab, tok, lane >> 1, (lane & 1) == 0, acc[t].x, other);
    }
  }

  // Stage the kTok x n_rows slice in shared memory, then write 16-byte vectors
  // to columns [s0, s0 + n_rows) of each ring slot.
  __syncthreads();
  __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(smem_raw);
#pragma unroll
  for (int t = 0; t < kT; ++t) {
    __nv_bfloat16* orow = os + (tok_row0 + t) * L::kWRows;
    orow[lane] = __float2bfloat16_rn(acc[t].x);
    if (!rope) orow[32 + lane] = __float2bfloat16_rn(acc[t].y);
  }
  __syncthreads();
  const int vec_per_row = n_rows / 8;
  for (int v = threadIdx.x; v < kTok * vec_per_row; v += L::kThreads) {
    const int t = v / vec_per_row, c = v - t * vec_per_row;
    const int tok = tok0 + t;
    if (tok < p.n_tok) {
      const int64_t slot = (p.slot0 + tok) % p.cap;
      const uint4 val = *reinterpret_cast<const uint4*>(os + t * L::kWRows + c * 8);
      *reinterpret_cast<uint4*>(p.cache + ((int64_t)b * p.cap + slot) * kRow + s0 + c * 8) = val;
    }
  }
}

template <int kDcT>
__global__ void __launch_bounds__(Slice<kDcT>::kThreads, 1)
    k_cache_append_slice(const __grid_constant__ AppendParams p, const __grid_constant__ RopeTable tab) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  if (blockIdx.z == Slice<kDcT>::kParts - 1) slice_body<kDcT, true>(p, tab, smem_raw);
  else slice_body<kDcT, false>(p, tab, smem_raw);
}

// ---- launch -----------------------------------------------------------------

template <class Kernel>
cudaError_t smem_attr(Kernel k, int bytes, bool (&done)[64], int dev) {
  if (dev < 0 || dev >= 64 || done[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

// The slice layout runs where all slices of all tiles fit in one wave: one CTA
// per SM, or (d_c >= 128, where a wide CTA takes longer than two slice CTAs
// sharing an SM) two per SM.  The tall layout runs where two of its CTAs fit on
// an SM and there are more tiles than SMs; everything else runs the wide layout.
template <int kDcT>
cudaError_t launch_cache_append_t(const AppendParams& p, int batch, int64_t t0, cudaStream_t stream) {
  using W = Wide<kDcT>;
  using T = Tall<kDcT>;
  using Sl = Slice<kDcT>;
  static bool wide_attr[64] = {false}, tall_attr[64] = {false}, slice_attr[64] = {false};
  static int tall_fit[64] = {0};      // 0 unknown, else 1 + (two tall CTAs fit on an SM)
  static int slice_fit[64] = {0};     // the same for slice CTAs
  static int sm_count[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t e = smem_attr(k_cache_append_wide<kDcT>, W::S::kSmemBytes, wide_attr, dev);
  if (e == cudaSuccess) e = smem_attr(k_cache_append_tall<kDcT>, T::S::kSmemBytes, tall_attr, dev);
  if (e == cudaSuccess) e = smem_attr(k_cache_append_slice<kDcT>, Sl::kSmemBytes, slice_attr, dev);
  if (e != cudaSuccess) return e;
  int sms = 148, fit2 = 0, slice_fit2 = 0;
  if (dev >= 0 && dev < 64) {
    if (sm_count[dev] == 0) {
      e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
    }
    if (tall_fit[dev] == 0) {
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_cache_append_tall<kDcT>, T::kThreads,
                                                        T::S::kSmemBytes);
      if (e != cudaSuccess) return e;
      tall_fit[dev] = 1 + (per_sm >= 2);
    }
    if (slice_fit[dev] == 0) {
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_cache_append_slice<kDcT>, Sl::kThreads,
                                                        Sl::kSmemBytes);
      if (e != cudaSuccess) return e;
      slice_fit[dev] = 1 + (per_sm >= 2);
    }
    sms = sm_count[dev];
    fit2 = tall_fit[dev] - 1;
    slice_fit2 = slice_fit[dev] - 1;
  }
  static thread_local RopeTable tab;
  static thread_local RopeTableKey tab_key;
  const int per_frame = p.grid_h * p.grid_w;
  build_rope_table(&tab, &tab_key, t0, (p.n_tok + per_frame - 1) / per_frame, p.grid_h, p.grid_w);
  dim3 grid((p.n_tok + kTok - 1) / kTok, batch);
  const int64_t tiles = (int64_t)grid.x * grid.y;
  const int64_t slices = tiles * Sl::kParts;
  if (slices <= sms || (kDcT >= 128 && slice_fit2 && slices <= 2 * (int64_t)sms))
    k_cache_append_slice<kDcT><<<dim3(grid.x, grid.y, Sl::kParts), Sl::kThreads, Sl::kSmemBytes, stream>>>(p, tab);
  else if (fit2 && tiles > sms)
    k_cache_append_tall<kDcT><<<grid, T::kThreads, T::S::kSmemBytes, stream>>>(p, tab);
  else
    k_cache_append_wide<kDcT><<<grid, W::kThreads, W::S::kSmemBytes, stream>>>(p, tab);
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
