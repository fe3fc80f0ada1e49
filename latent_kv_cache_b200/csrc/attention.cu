// Chunk attention over the latent KV cache (and the dense per-head baseline)
// on the sm_100a tensor cores.
//
// VideoMLA ("Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
// Diffusion", abstract; summary "Approach"): keys and values of every head are
// generated from one head-shared content latent c (192) plus one head-shared
// rope key k_r (32).  With W_UK absorbed into the query,
//     score(i, j) = scale * ( (q_h,i W_UK_h) . c_j + RoPE(q_r,h,i) . k_r,j ),
//     out_h,i     = ( sum_j softmax_j(score) c_j ) W_UV_h^T,
// so one CTA streams 224-wide cache rows [c ; k_r] and never materialises K or V.
//
// One CTA = one 128-query tile of one head of one sample; heads are the fastest
// grid index so the 12 CTAs that read the same cache tiles run together and
// share them through L2.  Warp roles (192 threads):
//   warp 0      TMA producer: q tile + W_UK_h, then [c ; k_r] tiles of 128 keys
//               into a 3-stage ring, then W_UV_h.
//   warp 1      TMEM allocation and the single MMA-issuing thread.
//   warps 2..5  softmax warpgroup; thread = query row = TMEM lane.
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,192)   O_lat accumulator (the prologue's q_abs lands here first)
//   [256,384) S buffer 0   (P, bf16, overwrites its first 64 columns)
//   [384,512) S buffer 1
//   epilogue: normalised O_lat as bf16 at [256,352), out accumulator at [384,512).
// Per key tile j the MMA thread issues S_j = Qa K_j^T (14 MMAs of K=16, the
// last two over the 64-byte-swizzled rope block) and then O += P_{j-1} C_{j-1}
// (8 MMAs, P read from tensor memory, C read MN-major from the same smem tile
// that served as K).  The softmax keeps the running max in log2 units and
// rescales O only when the max grows by more than 8 (2^8 headroom in bf16 P).
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;                // queries per tile
constexpr int kBN = 128;                // keys per tile
constexpr int kStages = 3;
constexpr uint32_t kBlk = 16384;        // 128 rows x 128 B (one 128B-swizzled block)
constexpr uint32_t kMlaStage = 3 * kBlk + 8192;   // [c: 3 blocks | k_r: 128 x 64 B]
constexpr uint32_t kDenseStage = 4 * kBlk;        // [K: 2 blocks | V: 2 blocks]
constexpr uint32_t kSmemBarOff = 229376;          // after Qa/Q + 3 stages (both kernels)
constexpr uint32_t kSmemBytes = kSmemBarOff + 256 + 1024;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS0 = 256;
constexpr uint32_t kTmemS1 = 384;
constexpr uint32_t kTmemOA = 256;
constexpr uint32_t kTmemOut = 384;

enum Bar {
  B_PRO = 0, B_QABS, B_QA,
  B_KVF0, B_KVF1, B_KVF2,
  B_KVE0, B_KVE1, B_KVE2,
  B_SF0, B_SF1,
  B_PF0, B_PF1,
  B_PV, B_OA, B_OUT, B_DRAIN,
  B_COUNT
};

struct ChunkMaps {
  CUtensorMap q;    // [B, Nq, H, 128] box (64, 1, 128, 1), 128B swizzle
  CUtensorMap wuk;  // [H*128, 192]    box (64, 128), 128B swizzle
  CUtensorMap wuv;  // [H*128, 192]    box (64, 128), 128B swizzle
  CUtensorMap c;    // [B, n_kv, 224]  box (64, 128, 1), 128B swizzle (content latent)
  CUtensorMap kr;   // [B, n_kv, 224]  box (32, 128, 1), 64B swizzle (rope key, x = 192)
};

struct DenseMaps {
  CUtensorMap q;  // [B, Nq, H, 128]
  CUtensorMap k;  // [B, Nk, H, 128]
  CUtensorMap v;  // [B, Nk, H, 128]
};

struct AttnParams {
  const uint16_t* q_rope;  // MLA only
  uint16_t* out;
  int* status;
  uint64_t wait_limit_ns;
  int64_t n_kv;
  int n_q;
  int heads;
  int n_kv_tiles;
  int grid_h;
  int grid_w;
  float scale_log2;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + 8u * i; }

// Bounded wait used when winding down after an abort (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                           int* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicCAS(status, 0, kDevTimeoutDrain);
      return;
    }
  }
}

// Bounded wait for the softmax warps: every lane waits, and the outcome is made
// warp-uniform so that the warp-collective tcgen05 instructions that follow are
// executed either by all 32 lanes or by none.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
  const bool ok = mbar_wait(bar, parity, ctl, kDevTimeoutSoftmax);
  return __all_sync(0xffffffffu, ok);
}

// Write 8 packed bf16x2 words (16 B chunks) of row r into a 128B-swizzled block.
__device__ __forceinline__ void st_sw128_chunk(uint8_t* blk, int r, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(blk + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
}
__device__ __forceinline__ void st_sw64_chunk(uint8_t* blk, int r, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(blk + r * 64 + ((chunk ^ ((r >> 1) & 3)) << 4)) = v;
}

// ---------------------------------------------------------------------------
// Softmax step for key tile j.  Returns false on abort.
// ---------------------------------------------------------------------------
template <int kOCols>
__device__ __forceinline__ bool softmax_tile(int j, uint32_t bars, uint32_t t_row,
                                             const AttnParams& p, const WaitCtl& ctl,
                                             float& m_run, float& l_run) {
  const int sb = j & 1;
  if (!warp_wait(bar_addr(bars, B_SF0 + sb), (j >> 1) & 1, ctl)) return false;
  tc_fence_after();
  const uint32_t scol = sb ? kTmemS1 : kTmemS0;
  float s[kBN];
  {
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(t_row + scol + 32 * c, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(r[e]);
    }
  }
  const int64_t kv0 = (int64_t)j * kBN;
  if (kv0 + kBN > p.n_kv) {
    const int valid = (int)(p.n_kv - kv0);
#pragma unroll
    for (int c = 0; c < kBN; ++c)
      if (c >= valid) s[c] = -INFINITY;
  }
  float mx = s[0];
#pragma unroll
  for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, s[c]);
  const float m_tile = mx * p.scale_log2;
  const bool need = m_tile > m_run + 8.0f;
  const float m_new = need ? m_tile : m_run;
  const float alpha = fast_exp2(m_run - m_new);
  float sum = 0.0f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 = fast_exp2(fmaf(s[32 * c + 2 * e], p.scale_log2, -m_new));
      const float p1 = fast_exp2(fmaf(s[32 * c + 2 * e + 1], p.scale_log2, -m_new));
      sum += p0 + p1;
      pk[e] = pack_bf16x2(p0, p1);
    }
    tmem_st16(t_row + scol + 16 * c, pk);
  }
  l_run = l_run * alpha + sum;
  if (j > 0) {
    // O may only be touched once the previous P.C product has landed.
    if (!warp_wait(bar_addr(bars, B_PV), (j - 1) & 1, ctl)) return false;
    if (__any_sync(0xffffffffu, need)) {
      tc_fence_after();
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < kOCols / 32; ++c) {
        tmem_ld32(t_row + kTmemO + 32 * c, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
        tmem_st32(t_row + kTmemO + 32 * c, r);
      }
    }
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(bar_addr(bars, B_PF0 + sb));
  m_run = m_new;
  return true;
}

// ---------------------------------------------------------------------------
// MLA chunk attention
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    k_chunk_attn(const __grid_constant__ ChunkMaps maps, const __grid_constant__ AttnParams p,
                 const __grid_constant__ RopeTable tab) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t qa = s_base;                 // Qa tile: 3 x 128B-swizzled blocks + rope block
  const uint32_t st0 = s_base + kMlaStage;    // stage s at st0 + s * kMlaStage
  const uint32_t bars = s_base + kSmemBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kSmemBarOff + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x % p.heads;
  const int q0 = (blockIdx.x / p.heads) * kBM;
  const int b = blockIdx.y;
  const int n_tiles = p.n_kv_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, B_PRO), 1);
    mbar_init(bar_addr(bars, B_QABS), 1);
    mbar_init(bar_addr(bars, B_QA), 128);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_addr(bars, B_KVF0 + s), 1);
      mbar_init(bar_addr(bars, B_KVE0 + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_addr(bars, B_SF0 + s), 1);
      mbar_init(bar_addr(bars, B_PF0 + s), 128);
    }
    mbar_init(bar_addr(bars, B_PV), 1);
    mbar_init(bar_addr(bars, B_OA), 128);
    mbar_init(bar_addr(bars, B_OUT), 1);
    mbar_init(bar_addr(bars, B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------- producer -------------------------------
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.wuk);
      tma_prefetch_desc(&maps.wuv);
      tma_prefetch_desc(&maps.c);
      tma_prefetch_desc(&maps.kr);
      const uint32_t st1 = st0 + kMlaStage;
      mbar_arrive_expect_tx(bar_addr(bars, B_PRO), 2 * kBlk + 3 * kBlk);
      tma_load_4d(st0, &maps.q, bar_addr(bars, B_PRO), 0, h, q0, b);
      tma_load_4d(st0 + kBlk, &maps.q, bar_addr(bars, B_PRO), 64, h, q0, b);
      tma_load_2d(st1, &maps.wuk, bar_addr(bars, B_PRO), 0, h * kDh);
      tma_load_2d(st1 + kBlk, &maps.wuk, bar_addr(bars, B_PRO), 64, h * kDh);
      tma_load_2d(st1 + 2 * kBlk, &maps.wuk, bar_addr(bars, B_PRO), 128, h * kDh);
      int last_use[kStages] = {-1, -1, -1};
      bool ok = true;
      for (int i = 0; i <= n_tiles; ++i) {
        const int st = i % kStages, use = i / kStages;
        const uint32_t sa = st0 + st * kMlaStage;
        if (use == 0) {
          if (st < 2) ok = mbar_wait(bar_addr(bars, B_QABS), 0, ctl, kDevTimeoutProducer);
        } else {
          ok = mbar_wait(bar_addr(bars, B_KVE0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer);
        }
        if (!ok) break;
        const uint32_t fb = bar_addr(bars, B_KVF0 + st);
        if (i < n_tiles) {
          const int kv0 = i * kBN;
          mbar_arrive_expect_tx(fb, kMlaStage);
          tma_load_3d(sa, &maps.c, fb, 0, kv0, b);
          tma_load_3d(sa + kBlk, &maps.c, fb, 64, kv0, b);
          tma_load_3d(sa + 2 * kBlk, &maps.c, fb, 128, kv0, b);
          tma_load_3d(sa + 3 * kBlk, &maps.kr, fb, kDc, kv0, b);
        } else {
          mbar_arrive_expect_tx(fb, 3 * kBlk);
          tma_load_2d(sa, &maps.wuv, fb, 0, h * kDh);
          tma_load_2d(sa + kBlk, &maps.wuv, fb, 64, h * kDh);
          tma_load_2d(sa + 2 * kBlk, &maps.wuv, fb, 128, h * kDh);
        }
        last_use[st] = use;
      }
      if (!ok) {
        // Let every copy already issued land before the CTA exits.
        drain_wait(bar_addr(bars, B_PRO), 0, p.wait_limit_ns, p.status);
        for (int s = 0; s < kStages; ++s)
          if (last_use[s] >= 0)
            drain_wait(bar_addr(bars, B_KVF0 + s), last_use[s] & 1, p.wait_limit_ns, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------- MMA ----------------------------------
      constexpr uint32_t kIdQabs = idesc_bf16_f32(128, 192, false, true);
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPv = idesc_bf16_f32(128, 192, false, true);
      constexpr uint32_t kIdOut = idesc_bf16_f32(128, 128, false, false);
      const uint32_t st1 = st0 + kMlaStage;
      bool ok = mbar_wait(bar_addr(bars, B_PRO), 0, ctl, kDevTimeoutMma);
      if (ok) {
        tc_fence_after();
        // q_abs = q_h . W_UK_h  (M 128, N 192, K 128); q K-major, W_UK MN-major.
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(st0 + (k >> 2) * kBlk + (k & 3) * 32, 16, 1024, kSw128);
          const uint64_t bd = smem_desc(st1 + k * 2048, kBlk, 1024, kSw128);
          umma_ss(tmem + kTmemO, a, bd, kIdQabs, k > 0);
        }
        umma_commit(bar_addr(bars, B_QABS));
        ok = mbar_wait(bar_addr(bars, B_QA), 0, ctl, kDevTimeoutMma);
      }
      auto issue_pv = [&](int jj) -> bool {
        if (!mbar_wait(bar_addr(bars, B_PF0 + (jj & 1)), (jj >> 1) & 1, ctl, kDevTimeoutMma))
          return false;
        tc_fence_after();
        const uint32_t sa = st0 + (jj % kStages) * kMlaStage;
        const uint32_t a_t = tmem + ((jj & 1) ? kTmemS1 : kTmemS0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bd = smem_desc(sa + k * 2048, kBlk, 1024, kSw128);
          umma_ts(tmem + kTmemO, a_t + k * 8, bd, kIdPv, (jj > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(bar_addr(bars, B_PV));
        umma_commit(bar_addr(bars, B_KVE0 + jj % kStages));
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kStages;
        ok = mbar_wait(bar_addr(bars, B_KVF0 + st), (j / kStages) & 1, ctl, kDevTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = st0 + st * kMlaStage;
        const uint32_t d = tmem + ((j & 1) ? kTmemS1 : kTmemS0);
#pragma unroll
        for (int k = 0; k < 14; ++k) {
          uint64_t a, bd;
          if (k < 12) {
            const uint32_t off = (k >> 2) * kBlk + (k & 3) * 32;
            a = smem_desc(qa + off, 16, 1024, kSw128);
            bd = smem_desc(sa + off, 16, 1024, kSw128);
          } else {
            const uint32_t off = 3 * kBlk + (k - 12) * 32;
            a = smem_desc(qa + off, 16, 512, kSw64);
            bd = smem_desc(sa + off, 16, 512, kSw64);
          }
          umma_ss(d, a, bd, kIdS, k > 0);
        }
        umma_commit(bar_addr(bars, B_SF0 + (j & 1)));
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) ok = issue_pv(n_tiles - 1);
      if (ok) {
        const int st = n_tiles % kStages;
        ok = mbar_wait(bar_addr(bars, B_KVF0 + st), (n_tiles / kStages) & 1, ctl, kDevTimeoutMma) &&
             mbar_wait(bar_addr(bars, B_OA), 0, ctl, kDevTimeoutMma);
        if (ok) {
          tc_fence_after();
          const uint32_t sa = st0 + st * kMlaStage;
          // out = O_lat/l . W_UV_h^T  (M 128, N 128, K 192); A from TMEM, W_UV K-major.
#pragma unroll
          for (int k = 0; k < 12; ++k) {
            const uint64_t bd = smem_desc(sa + (k >> 2) * kBlk + (k & 3) * 32, 16, 1024, kSw128);
            umma_ts(tmem + kTmemOut, tmem + kTmemOA + k * 8, bd, kIdOut, k > 0);
          }
          umma_commit(bar_addr(bars, B_OUT));
        }
      }
      if (!ok) {
        umma_commit(bar_addr(bars, B_DRAIN));
        drain_wait(bar_addr(bars, B_DRAIN), 0, p.wait_limit_ns, p.status);
      }
    }
  } else {
    // -------------------------------- softmax ---------------------------------
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t t_row = tmem + ((uint32_t)(qd * 32) << 16);
    const int qi = q0 + r;
    bool ok = warp_wait(bar_addr(bars, B_QABS), 0, ctl);
    if (ok) {
      tc_fence_after();
      uint8_t* qa_p = smem;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 6; ++c) {
        tmem_ld32(t_row + kTmemO + 32 * c, v);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7]));
          st_sw128_chunk(qa_p + (c >> 1) * kBlk, r, (c & 1) * 4 + q4, w);
        }
      }
      // Rope part of the query, rotated with the query's own (t, row, col).
      float qr[kDr];
#pragma unroll
      for (int e = 0; e < kDr; ++e) qr[e] = 0.0f;
      if (qi < p.n_q) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.q_rope + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDr);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 u = __ldg(src + c);
          qr[8 * c + 0] = bf16lo_to_f32(u.x); qr[8 * c + 1] = bf16hi_to_f32(u.x);
          qr[8 * c + 2] = bf16lo_to_f32(u.y); qr[8 * c + 3] = bf16hi_to_f32(u.y);
          qr[8 * c + 4] = bf16lo_to_f32(u.z); qr[8 * c + 5] = bf16hi_to_f32(u.z);
          qr[8 * c + 6] = bf16lo_to_f32(u.w); qr[8 * c + 7] = bf16hi_to_f32(u.w);
        }
        const int per_frame = p.grid_h * p.grid_w;
        const int f = qi / per_frame;
        const int rem = qi - f * per_frame;
        const int row = rem / p.grid_w;
        const int col = rem - row * p.grid_w;
#pragma unroll
        for (int pr = 0; pr < kDr / 2; ++pr) {
          float2 cs;
          if (pr < kPairsT) cs = tab.t[f][pr];
          else if (pr < kPairsT + kPairsH) cs = tab.h[row][pr - kPairsT];
          else cs = tab.w[col][pr - kPairsT - kPairsH];
          const float a = qr[2 * pr], bb = qr[2 * pr + 1];
          qr[2 * pr] = a * cs.x - bb * cs.y;
          qr[2 * pr + 1] = a * cs.y + bb * cs.x;
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 w;
        w.x = pack_bf16x2(qr[8 * c + 0], qr[8 * c + 1]);
        w.y = pack_bf16x2(qr[8 * c + 2], qr[8 * c + 3]);
        w.z = pack_bf16x2(qr[8 * c + 4], qr[8 * c + 5]);
        w.w = pack_bf16x2(qr[8 * c + 6], qr[8 * c + 7]);
        st_sw64_chunk(qa_p + 3 * kBlk, r, c, w);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_addr(bars, B_QA));
    }
    float m_run = -INFINITY, l_run = 0.0f;
    for (int j = 0; ok && j < n_tiles; ++j) ok = softmax_tile<kDc>(j, bars, t_row, p, ctl, m_run, l_run);
    if (ok) ok = warp_wait(bar_addr(bars, B_PV), (n_tiles - 1) & 1, ctl);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 6; ++c) {
        tmem_ld32(t_row + kTmemO + 32 * c, v);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv_l, __uint_as_float(v[2 * e + 1]) * inv_l);
        tmem_st16(t_row + kTmemOA + 16 * c, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(bars, B_OA));
      ok = warp_wait(bar_addr(bars, B_OUT), 0, ctl);
      if (ok) {
        tc_fence_after();
        uint4* dst = reinterpret_cast<uint4*>(p.out + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDh);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(t_row + kTmemOut + 32 * c, v);
          tmem_ld_wait();
          if (qi < p.n_q) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1]));
              w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3]));
              w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5]));
              w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7]));
              dst[4 * c + q4] = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Dense per-head attention (d = 128), same skeleton without the projections
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    k_dense_attn(const __grid_constant__ DenseMaps maps, const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t qs = s_base;                 // Q tile: 2 x 128B-swizzled blocks
  const uint32_t st0 = s_base + 2 * kBlk;     // stage s at st0 + s * kDenseStage
  const uint32_t bars = s_base + kSmemBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kSmemBarOff + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x % p.heads;
  const int q0 = (blockIdx.x / p.heads) * kBM;
  const int b = blockIdx.y;
  const int n_tiles = p.n_kv_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, B_PRO), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_addr(bars, B_KVF0 + s), 1);
      mbar_init(bar_addr(bars, B_KVE0 + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_addr(bars, B_SF0 + s), 1);
      mbar_init(bar_addr(bars, B_PF0 + s), 128);
    }
    mbar_init(bar_addr(bars, B_PV), 1);
    mbar_init(bar_addr(bars, B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      mbar_arrive_expect_tx(bar_addr(bars, B_PRO), 2 * kBlk);
      tma_load_4d(qs, &maps.q, bar_addr(bars, B_PRO), 0, h, q0, b);
      tma_load_4d(qs + kBlk, &maps.q, bar_addr(bars, B_PRO), 64, h, q0, b);
      int last_use[kStages] = {-1, -1, -1};
      bool ok = true;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % kStages, use = i / kStages;
        const uint32_t sa = st0 + st * kDenseStage;
        if (use > 0) ok = mbar_wait(bar_addr(bars, B_KVE0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer);
        if (!ok) break;
        const uint32_t fb = bar_addr(bars, B_KVF0 + st);
        const int kv0 = i * kBN;
        mbar_arrive_expect_tx(fb, kDenseStage);
        tma_load_4d(sa, &maps.k, fb, 0, h, kv0, b);
        tma_load_4d(sa + kBlk, &maps.k, fb, 64, h, kv0, b);
        tma_load_4d(sa + 2 * kBlk, &maps.v, fb, 0, h, kv0, b);
        tma_load_4d(sa + 3 * kBlk, &maps.v, fb, 64, h, kv0, b);
        last_use[st] = use;
      }
      if (!ok) {
        drain_wait(bar_addr(bars, B_PRO), 0, p.wait_limit_ns, p.status);
        for (int s = 0; s < kStages; ++s)
          if (last_use[s] >= 0)
            drain_wait(bar_addr(bars, B_KVF0 + s), last_use[s] & 1, p.wait_limit_ns, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPv = idesc_bf16_f32(128, 128, false, true);
      bool ok = mbar_wait(bar_addr(bars, B_PRO), 0, ctl, kDevTimeoutMma);
      auto issue_pv = [&](int jj) -> bool {
        if (!mbar_wait(bar_addr(bars, B_PF0 + (jj & 1)), (jj >> 1) & 1, ctl, kDevTimeoutMma))
          return false;
        tc_fence_after();
        const uint32_t sv = st0 + (jj % kStages) * kDenseStage + 2 * kBlk;
        const uint32_t a_t = tmem + ((jj & 1) ? kTmemS1 : kTmemS0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bd = smem_desc(sv + k * 2048, kBlk, 1024, kSw128);
          umma_ts(tmem + kTmemO, a_t + k * 8, bd, kIdPv, (jj > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(bar_addr(bars, B_PV));
        umma_commit(bar_addr(bars, B_KVE0 + jj % kStages));
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kStages;
        ok = mbar_wait(bar_addr(bars, B_KVF0 + st), (j / kStages) & 1, ctl, kDevTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = st0 + st * kDenseStage;
        const uint32_t d = tmem + ((j & 1) ? kTmemS1 : kTmemS0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * kBlk + (k & 3) * 32;
          umma_ss(d, smem_desc(qs + off, 16, 1024, kSw128), smem_desc(sa + off, 16, 1024, kSw128),
                  kIdS, k > 0);
        }
        umma_commit(bar_addr(bars, B_SF0 + (j & 1)));
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) ok = issue_pv(n_tiles - 1);
      if (!ok) {
        umma_commit(bar_addr(bars, B_DRAIN));
        drain_wait(bar_addr(bars, B_DRAIN), 0, p.wait_limit_ns, p.status);
      }
    }
  } else {
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t t_row = tmem + ((uint32_t)(qd * 32) << 16);
    const int qi = q0 + r;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; ok && j < n_tiles; ++j) ok = softmax_tile<kDh>(j, bars, t_row, p, ctl, m_run, l_run);
    if (ok) ok = warp_wait(bar_addr(bars, B_PV), (n_tiles - 1) & 1, ctl);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      uint4* dst = reinterpret_cast<uint4*>(p.out + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDh);
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(t_row + kTmemO + 32 * c, v);
        tmem_ld_wait();
        if (qi < p.n_q) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv_l, __uint_as_float(v[8 * q4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv_l, __uint_as_float(v[8 * q4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv_l, __uint_as_float(v[8 * q4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv_l, __uint_as_float(v[8 * q4 + 7]) * inv_l);
            dst[4 * c + q4] = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 tensor map; dims innermost first; strides in bytes for dims 1..rank-1.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t elem[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
                  strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool set_smem_attr(const void* fn, bool* done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

bool make_qmap(CUtensorMap* m, const uint16_t* q, int batch, int n_rows, int heads) {
  const cuuint64_t dims[4] = {(cuuint64_t)kDh, (cuuint64_t)heads, (cuuint64_t)n_rows, (cuuint64_t)batch};
  const cuuint64_t strides[3] = {(cuuint64_t)kDh * 2, (cuuint64_t)heads * kDh * 2,
                                 (cuuint64_t)n_rows * heads * kDh * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBM, 1};
  return make_map(m, q, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_chunk_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                   const uint16_t* w_uv, const uint16_t* cache, int batch, int n_q,
                                   int heads, int64_t cap, int64_t n_kv, int64_t t0, int grid_h,
                                   int grid_w, float scale, uint16_t* out, int* status,
                                   cudaStream_t stream, bool* encode_failed) {
  static bool attr_done[64] = {false};
  *encode_failed = false;
  if (!set_smem_attr((const void*)k_chunk_attn, attr_done)) return cudaErrorInvalidValue;
  ChunkMaps maps;
  bool ok = make_qmap(&maps.q, q, batch, n_q, heads);
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kDc, (cuuint64_t)heads * kDh};
    const cuuint64_t strides[1] = {(cuuint64_t)kDc * 2};
    const cuuint32_t box[2] = {64, 128};
    ok = ok && make_map(&maps.wuk, w_uk, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&maps.wuv, w_uv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kDrow, (cuuint64_t)n_kv, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)kDrow * 2, (cuuint64_t)cap * kDrow * 2};
    const cuuint32_t box_c[3] = {64, (cuuint32_t)kBN, 1};
    const cuuint32_t box_r[3] = {32, (cuuint32_t)kBN, 1};
    ok = ok && make_map(&maps.c, cache, 3, dims, strides, box_c, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&maps.kr, cache, 3, dims, strides, box_r, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnParams p{};
  p.q_rope = q_rope;
  p.out = out;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  p.n_kv = n_kv;
  p.n_q = n_q;
  p.heads = heads;
  p.n_kv_tiles = (int)((n_kv + kBN - 1) / kBN);
  p.grid_h = grid_h;
  p.grid_w = grid_w;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  static thread_local RopeTable tab;
  const int per_frame = grid_h * grid_w;
  build_rope_table(&tab, t0, (n_q + per_frame - 1) / per_frame, grid_h, grid_w);
  dim3 grid((unsigned)(((n_q + kBM - 1) / kBM) * heads), (unsigned)batch);
  k_chunk_attn<<<grid, kThreads, kSmemBytes, stream>>>(maps, p, tab);
  return cudaGetLastError();
}

cudaError_t launch_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int batch,
                                   int n_q, int64_t n_kv, int heads, float scale, uint16_t* out,
                                   int* status, cudaStream_t stream, bool* encode_failed) {
  static bool attr_done[64] = {false};
  *encode_failed = false;
  if (!set_smem_attr((const void*)k_dense_attn, attr_done)) return cudaErrorInvalidValue;
  DenseMaps maps;
  bool ok = make_qmap(&maps.q, q, batch, n_q, heads) && make_qmap(&maps.k, k, batch, (int)n_kv, heads) &&
            make_qmap(&maps.v, v, batch, (int)n_kv, heads);
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnParams p{};
  p.out = out;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  p.n_kv = n_kv;
  p.n_q = n_q;
  p.heads = heads;
  p.n_kv_tiles = (int)((n_kv + kBN - 1) / kBN);
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  dim3 grid((unsigned)(((n_q + kBM - 1) / kBM) * heads), (unsigned)batch);
  k_dense_attn<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace vmla
