// Per-head keys and values materialised from the latent cache:
//     K_h[j] = c_j . W_UK_h^T,   V_h[j] = c_j . W_UV_h^T      (128 values each)
// for every cached token j and head h.  This is the non-absorbed form of
// VideoMLA's latent attention ("Low-Rank Latent KV Cache for Minute-Scale
// Autoregressive Video Diffusion", abstract: per-head keys and values are
// generated from the head-shared content latent).  Done once per layer and
// chunk, it lets every denoising step of that chunk run a d = 128 + 32
// attention over explicit keys instead of the absorbed d = 224 + 192 one.
//
// One CTA = 128 keys x one head: D[128 x 256] = C[128 x 192] . [W_UK_h ; W_UV_h]^T
// (12 tcgen05 MMAs, N = 256, operands staged by TMA), then a bf16 epilogue that
// writes K_h to heads [0, H) and V_h to heads [H, 2H) of kv[B, n_kv, 2H, 128].
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 128;
constexpr uint32_t kBlk = 128 * 128;        // 128 rows x 128 B, 128B swizzle
constexpr uint32_t kA = 0;                  // C tile: 3 blocks (latent 0-63, 64-127, 128-191)
constexpr uint32_t kB = 3 * kBlk;           // [W_UK_h ; W_UV_h]: per latent block 256 rows
constexpr uint32_t kBBlk = 2 * kBlk;        // one latent block of B (256 rows)
constexpr uint32_t kBar = kB + 3 * kBBlk;   // 147456
constexpr uint32_t kSmemBytes = kBar + 64 + 1024;
constexpr uint32_t kTmemCols = 256;

struct MatParams {
  uint16_t* kv;  // [B, n_kv, 2H, 128]
  int* status;
  uint64_t wait_limit_ns;
  int64_t n_kv;
  int heads;
};

struct MatGemmMaps {
  CUtensorMap c;    // cache [B, n_kv, 224] box (64, 128, 1), 128B swizzle
  CUtensorMap wuk;  // [H*128, 192] box (64, 128), 128B swizzle
  CUtensorMap wuv;
};

__global__ void __launch_bounds__(kThreads, 1)
    k_materialize_kv(const __grid_constant__ MatGemmMaps maps, const __grid_constant__ MatParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uint32_t pad = (uint32_t)(((raw + 1023) & ~uintptr_t(1023)) - raw);
  uint8_t* smem = smem_raw + pad;  // kSmemBytes reserves 1024 B of slack for this
  const uint32_t base = smem_u32(smem);
  const uint32_t bar_full = base + kBar, bar_mma = base + kBar + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kBar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBar + 20);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kv0 = blockIdx.x * 128;
  const int h = blockIdx.y;
  const int b = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_full, 3 * kBlk + 3 * kBBlk);
#pragma unroll
    for (int blk = 0; blk < 3; ++blk) {
      tma_load_3d(base + kA + blk * kBlk, &maps.c, bar_full, 64 * blk, kv0, b);
      tma_load_2d(base + kB + blk * kBBlk, &maps.wuk, bar_full, 64 * blk, h * kDh);
      tma_load_2d(base + kB + blk * kBBlk + kBlk, &maps.wuv, bar_full, 64 * blk, h * kDh);
    }
    ok = mbar_wait(bar_full, 0, ctl, kDevTimeoutMma);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t kId = idesc_bf16_f32(128, 256, false, false);
#pragma unroll
      for (int k = 0; k < 12; ++k) {
        const uint32_t off = (k & 3) * 32;
        const uint64_t a = smem_desc(base + kA + (k >> 2) * kBlk + off, 16, 1024, kSw128);
        const uint64_t bd = smem_desc(base + kB + (k >> 2) * kBBlk + off, 16, 1024, kSw128);
        umma_ss(tmem, a, bd, kId, k > 0);
      }
      umma_commit(bar_mma);
    } else {
      // The copies issued above must land before the CTA exits.
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_full, 0) && globaltimer_ns() - t0 < p.wait_limit_ns) {
      }
    }
  }
  // Epilogue: thread = key row; TMEM lanes of warp w are rows 32 w .. 32 w + 31.
  const bool ok_all = mbar_wait(bar_mma, 0, ctl, kDevTimeoutSoftmax);
  if (__all_sync(0xffffffffu, ok_all)) {
    tc_fence_after();
    const int r = warp * 32 + lane;
    const int64_t j = (int64_t)kv0 + r;
    const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t v[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {  // columns 0-127: K_h, 128-255: V_h
      tmem_ld32(t_row + 32 * c, v);
      tmem_ld_wait();
      if (j < p.n_kv) {
        const int head = c < 4 ? h : p.heads + h;
        uint4* dst = reinterpret_cast<uint4*>(
            p.kv + (((int64_t)b * p.n_kv + j) * (2 * p.heads) + head) * kDh + 32 * (c & 3));
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7]));
          dst[q4] = w;
        }
      }
    }
  } else if (threadIdx.x == 0 && ok) {
    // MMAs were issued but the epilogue gave up: let them finish before TMEM is freed.
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar_mma, 0) && globaltimer_ns() - t0 < p.wait_limit_ns) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  cuuint32_t elem[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box,
            elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_materialize_kv(const uint16_t* w_uk, const uint16_t* w_uv, const uint16_t* cache, int batch,
                                  int heads, int64_t cap, int64_t n_kv, uint16_t* kv, int* status,
                                  cudaStream_t stream, bool* encode_failed) {
  static bool attr_done[64] = {false};
  *encode_failed = false;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_materialize_kv, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  MatGemmMaps maps;
  bool ok;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kDrow, (cuuint64_t)n_kv, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)kDrow * 2, (cuuint64_t)cap * kDrow * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    ok = encode(&maps.c, cache, 3, dims, strides, box);
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kDc, (cuuint64_t)heads * kDh};
    const cuuint64_t strides[1] = {(cuuint64_t)kDc * 2};
    const cuuint32_t box[2] = {64, 128};
    ok = ok && encode(&maps.wuk, w_uk, 2, dims, strides, box) && encode(&maps.wuv, w_uv, 2, dims, strides, box);
  }
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  MatParams p{kv, status, kWaitLimitNs, n_kv, heads};
  dim3 grid((unsigned)((n_kv + 127) / 128), (unsigned)heads, (unsigned)batch);
  k_materialize_kv<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace vmla
