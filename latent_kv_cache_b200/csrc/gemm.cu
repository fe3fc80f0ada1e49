// bf16 GEMM on the tensor cores for the projections either side of the latent
// attention: C[M x N] = A[M x K] . B[N x K]^T (nn.Linear weights), fp32
// accumulation in TMEM, bf16 output.  The N columns come from two weight matrices
// (B0 rows [0, N0), B1 rows [N0, N0 + N1)) written to two outputs, so the query
// and rope-query projections share one pass over the hidden states:
//     q   = x . W_Q^T    [tokens, H*128]
//     q_r = x . W_QR^T   [tokens, H*32]   (RoPE3D is applied by the attention kernel)
// and the output projection is the one-matrix case  y = o . W_O^T.
//
// One CTA = a 128 x 256 tile (N = 256 MMAs, the efficient tcgen05 shape);
// 192 threads: warp 0 TMA producer (4-stage ring of [A 128x64 | B 256x64]
// 128B-swizzled k blocks), warp 1 TMEM allocation + MMA issue, warps 2-5 the
// epilogue (TMEM lane = output row).
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr uint32_t kABytes = kBM * kBK * 2;           // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;           // 32 KB (two 128-row halves)
constexpr uint32_t kStageBytes = kABytes + kBBytes;   // 48 KB
constexpr uint32_t kBarOff = kStages * kStageBytes;   // 196608
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kTmemCols = 256;

enum { G_FULL0 = 0, G_EMPTY0 = kStages, G_DONE = 2 * kStages, G_DRAIN, G_COUNT };

struct GemmMaps {
  CUtensorMap a;   // [M, K] box (64, 128)
  CUtensorMap b0;  // [N0, K] box (64, 128)
  CUtensorMap b1;  // [N1, K] box (64, 128) (a copy of b0 when N1 == 0)
};

struct GemmParams {
  uint16_t* c0;
  uint16_t* c1;
  int64_t ldc0, ldc1;
  int m, n0, n1, k;
  int* status;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ uint32_t gbar(uint32_t base, int i) { return base + 8u * i; }

__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_bf16(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~uintptr_t(1023)) - raw);  // kSmemBytes keeps 1 KB of slack
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + kBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * G_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;
  const int n0 = blockIdx.y * kBN;
  const int nk = p.k / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(gbar(bars, G_FULL0 + s), 1);
      mbar_init(gbar(bars, G_EMPTY0 + s), 1);
    }
    mbar_init(gbar(bars, G_DONE), 1);
    mbar_init(gbar(bars, G_DRAIN), 1);
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
      tma_prefetch_desc(&maps.a);
      tma_prefetch_desc(&maps.b0);
      tma_prefetch_desc(&maps.b1);
      int last_use[kStages] = {-1, -1, -1, -1};
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % kStages, use = kb / kStages;
        if (use > 0 && !(ok = mbar_wait(gbar(bars, G_EMPTY0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer)))
          break;
        const uint32_t sa = base + st * kStageBytes, fb = gbar(bars, G_FULL0 + st);
        mbar_arrive_expect_tx(fb, kStageBytes);
        tma_load_2d(sa, &maps.a, fb, kb * kBK, m0);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // each 128-row half of the tile comes from B0 or B1
          const int row = n0 + 128 * half;
          const uint32_t dst = sa + kABytes + half * (kBBytes / 2);
          if (row < p.n0) tma_load_2d(dst, &maps.b0, fb, kb * kBK, row);
          else tma_load_2d(dst, &maps.b1, fb, kb * kBK, row - p.n0);
        }
        last_use[st] = use;
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s) {
          if (last_use[s] < 0) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(gbar(bars, G_FULL0 + s), last_use[s] & 1) &&
                 globaltimer_ns() - t0 < p.wait_limit_ns) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(kBM, kBN, false, false);
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int st = kb % kStages;
        ok = mbar_wait(gbar(bars, G_FULL0 + st), (kb / kStages) & 1, ctl, kDevTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = base + st * kStageBytes;
        const uint64_t a0 = smem_desc(sa, 16, 1024, kSw128);
        const uint64_t b0 = smem_desc(sa + kABytes, 16, 1024, kSw128);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)  // +32 bytes = +2 in the descriptor's address field
          umma_ss(tmem, a0 + 2u * k, b0 + 2u * k, kId, (kb > 0 || k > 0) ? 1u : 0u);
        umma_commit(gbar(bars, G_EMPTY0 + st));
      }
      if (ok) {
        umma_commit(gbar(bars, G_DONE));
      } else {
        umma_commit(gbar(bars, G_DRAIN));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(gbar(bars, G_DRAIN), 0) && globaltimer_ns() - t0 < p.wait_limit_ns) {
        }
      }
    }
  } else {
    // Epilogue warps 2..5: TMEM lane quadrant = warp % 4, row = 32 * quadrant + lane.
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const int row = m0 + r;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(gbar(bars, G_DONE), 0, ctl, kDevTimeoutSoftmax));
    if (ok) {
      tc_fence_after();
      const uint32_t t_row = tmem + ((uint32_t)(qd * 32) << 16);
      uint32_t v[32];
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        tmem_ld32(t_row + 32 * c, v);
        tmem_ld_wait();
        const int col = n0 + 32 * c;  // 32 columns never straddle N0 (a multiple of 128)
        if (row < p.m && col < p.n0 + p.n1) {
          uint16_t* dst = col < p.n0 ? p.c0 + (int64_t)row * p.ldc0 + col
                                     : p.c1 + (int64_t)row * p.ldc1 + (col - p.n0);
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1]));
            w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3]));
            w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5]));
            w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7]));
            d4[q4] = w;
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [rows, cols] bf16 row-major, box 64 columns x 128 rows, 128B swizzle.
bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t elem[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// C0[m, n0] (row stride ldc0) and C1[m, n1] (ldc1) from A[m, k] . [B0 ; B1]^T.
// Requires k % 64 == 0, n0 % 128 == 0, n1 % 32 == 0, 16-byte aligned pointers and strides.
cudaError_t launch_gemm_pair(const uint16_t* a, const uint16_t* b0, const uint16_t* b1, int m, int n0, int n1,
                             int k, uint16_t* c0, int64_t ldc0, uint16_t* c1, int64_t ldc1, int* status,
                             cudaStream_t stream, bool* encode_failed) {
  static bool attr_done[64] = {false};
  *encode_failed = false;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  GemmMaps maps;
  bool ok = encode_rows(&maps.a, a, m, k) && encode_rows(&maps.b0, b0, n0, k);
  ok = ok && (n1 > 0 ? encode_rows(&maps.b1, b1, n1, k) : encode_rows(&maps.b1, b0, n0, k));
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  GemmParams p{c0, n1 > 0 ? c1 : c0, ldc0, n1 > 0 ? ldc1 : ldc0, m, n0, n1, k, status, kWaitLimitNs};
  dim3 grid((unsigned)((m + kBM - 1) / kBM), (unsigned)((n0 + n1 + kBN - 1) / kBN));
  k_gemm_bf16<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace vmla
