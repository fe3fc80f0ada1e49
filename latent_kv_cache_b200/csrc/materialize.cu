// Per-head keys and values materialised from the latent cache:
//     K_h[j] = c_j . W_UK_h^T,   V_h[j] = c_j . W_UV_h^T      (128 values each)
// for every cached token j and head h.  This is the non-absorbed form of
// VideoMLA's latent attention ("Low-Rank Latent KV Cache for Minute-Scale
// Autoregressive Video Diffusion", abstract: per-head keys and values are
// generated from the head-shared content latent).  Done once per layer and
// chunk, it lets every denoising step of that chunk run a d = 128 + 32
// attention over explicit keys instead of the absorbed d = 224 + 192 one.
//
// Persistent kernel: CTA g takes a contiguous range of work items (sample, head,
// 128-key tile), ordered head-major so W_UK_h / W_UV_h are loaded once per head
// and stay in shared memory.  Per item: D[128 keys x 256] = C[128 x 192] .
// [W_UK_h ; W_UV_h]^T (12 tcgen05 MMAs, N = 256), then a bf16 epilogue that
// writes K_h to heads [0, H) and V_h to heads [H, 2H) of kv[B, n_kv, 2H, 128].
// 192 threads: warp 0 TMA producer (the C tiles through a 2-stage ring, W at each
// head change), warp 1 TMEM allocation + the MMA thread, warps 2-5 the epilogue.
// TMEM holds two 256-column accumulators, so an item's stores overlap the next
// item's MMAs.  The epilogue stages each 64-column block of its 32 rows in shared
// memory and writes it back four full 128-byte lines per store instruction.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 192;
constexpr int kCStages = 2;
constexpr uint32_t kBlk = 128 * 128;        // 128 rows x 128 B, 128B swizzle
constexpr uint32_t kCBytes = 3 * kBlk;      // C tile: 3 blocks (latent 0-63, 64-127, 128-191)
constexpr uint32_t kBBlk = 2 * kBlk;        // one latent block of [W_UK_h ; W_UV_h] (256 rows)
constexpr uint32_t kW = 0;                  // W: 3 latent blocks of 256 rows
constexpr uint32_t kC0 = 3 * kBBlk;         // C ring
constexpr uint32_t kBar = kC0 + kCStages * kCBytes;  // 196608
// Epilogue staging: per epilogue warp, 32 rows x 64 bf16 (128 B) padded to 144 B
// so that row-per-lane writes hit distinct banks.
constexpr uint32_t kStgRow = 144;
constexpr uint32_t kStgWarp = 32 * kStgRow;
constexpr uint32_t kStg = kBar + 256;
constexpr uint32_t kSmemBytes = kStg + 4 * kStgWarp + 1024;
constexpr uint32_t kTmemCols = 512;         // two 256-column accumulators

enum {
  M_CFULL0 = 0, M_CEMPTY0 = kCStages, M_WFULL = 2 * kCStages, M_WEMPTY, M_ACCF0, M_ACCE0 = M_ACCF0 + 2,
  M_DRAIN = M_ACCE0 + 2, M_COUNT
};
static_assert(8 * M_COUNT + 8 <= 256, "barrier area");

struct MatParams {
  uint16_t* kv;  // [B, n_kv, 2H, 128]
  int* status;
  uint64_t wait_limit_ns;
  int64_t n_kv;
  int heads;
  int n_tiles;   // key tiles per (sample, head)
  int n_items;   // batch * heads * n_tiles
};

struct MatGemmMaps {
  CUtensorMap c;    // cache [B, n_kv, 224] box (64, 128, 1), 128B swizzle
  CUtensorMap wuk;  // [H*128, 192] box (64, 128), 128B swizzle
  CUtensorMap wuv;
};

__device__ __forceinline__ uint32_t mbar(uint32_t base, int i) { return base + 8u * i; }

__global__ void __launch_bounds__(kThreads, 1)
    k_materialize_kv(const __grid_constant__ MatGemmMaps maps, const __grid_constant__ MatParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uint32_t pad = (uint32_t)(((raw + 1023) & ~uintptr_t(1023)) - raw);
  uint8_t* smem = smem_raw + pad;  // kSmemBytes reserves 1024 B of slack for this
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + kBar;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kBar + 8 * M_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // This CTA's items: [it0, it1), item = ((b * heads + h) * n_tiles + tile).
  const int it0 = (int)((int64_t)p.n_items * blockIdx.x / gridDim.x);
  const int it1 = (int)((int64_t)p.n_items * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCStages; ++s) {
      mbar_init(mbar(bars, M_CFULL0 + s), 1);
      mbar_init(mbar(bars, M_CEMPTY0 + s), 1);
    }
    mbar_init(mbar(bars, M_WFULL), 1);
    mbar_init(mbar(bars, M_WEMPTY), 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(mbar(bars, M_ACCF0 + a), 1);
      mbar_init(mbar(bars, M_ACCE0 + a), 4);  // one arrival per epilogue warp
    }
    mbar_init(mbar(bars, M_DRAIN), 1);
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
      // ------------------------------ producer ------------------------------
      tma_prefetch_desc(&maps.c);
      tma_prefetch_desc(&maps.wuk);
      tma_prefetch_desc(&maps.wuv);
      int last_c[kCStages] = {-1, -1};
      int wloads = 0, cur_bh = -1;
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        const int bh = it / p.n_tiles, tile = it - bh * p.n_tiles;
        const int b = bh / p.heads, h = bh - b * p.heads;
        if (bh != cur_bh) {  // new head: W_UK_h / W_UV_h, once the old ones are no longer read
          if (wloads > 0 && !(ok = mbar_wait(mbar(bars, M_WEMPTY), (wloads - 1) & 1, ctl, kDevTimeoutProducer)))
            break;
          const uint32_t wb = mbar(bars, M_WFULL);
          mbar_arrive_expect_tx(wb, 3 * kBBlk);
#pragma unroll
          for (int blk = 0; blk < 3; ++blk) {
            tma_load_2d(base + kW + blk * kBBlk, &maps.wuk, wb, 64 * blk, h * kDh);
            tma_load_2d(base + kW + blk * kBBlk + kBlk, &maps.wuv, wb, 64 * blk, h * kDh);
          }
          ++wloads;
          cur_bh = bh;
        }
        const int i = it - it0, st = i % kCStages, use = i / kCStages;
        if (use > 0 && !(ok = mbar_wait(mbar(bars, M_CEMPTY0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer)))
          break;
        const uint32_t fb = mbar(bars, M_CFULL0 + st);
        mbar_arrive_expect_tx(fb, kCBytes);
#pragma unroll
        for (int blk = 0; blk < 3; ++blk)
          tma_load_3d(base + kC0 + st * kCBytes + blk * kBlk, &maps.c, fb, 64 * blk, tile * 128, b);
        last_c[st] = use;
      }
      if (!ok) {  // copies already issued must land before the CTA exits
        if (wloads > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(mbar(bars, M_WFULL), (wloads - 1) & 1) && globaltimer_ns() - t0 < p.wait_limit_ns) {
          }
        }
        for (int s = 0; s < kCStages; ++s) {
          if (last_c[s] < 0) continue;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(mbar(bars, M_CFULL0 + s), last_c[s] & 1) && globaltimer_ns() - t0 < p.wait_limit_ns) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------- MMA --------------------------------
      constexpr uint32_t kId = idesc_bf16_f32(128, 256, false, false);
      int wsegs = 0, cur_bh = -1;
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        const int i = it - it0, st = i % kCStages, acc = i & 1;
        const int bh = it / p.n_tiles;
        if (bh != cur_bh) {
          if (!(ok = mbar_wait(mbar(bars, M_WFULL), wsegs & 1, ctl, kDevTimeoutMma))) break;
          ++wsegs;
          cur_bh = bh;
        }
        if (i >= 2 && !(ok = mbar_wait(mbar(bars, M_ACCE0 + acc), ((i >> 1) - 1) & 1, ctl, kDevTimeoutMma))) break;
        if (!(ok = mbar_wait(mbar(bars, M_CFULL0 + st), (i / kCStages) & 1, ctl, kDevTimeoutMma))) break;
        tc_fence_after();
        const uint32_t cs = base + kC0 + st * kCBytes;
#pragma unroll
        for (int k = 0; k < 12; ++k) {
          const uint32_t off = (k & 3) * 32;
          const uint64_t a = smem_desc(cs + (k >> 2) * kBlk + off, 16, 1024, kSw128);
          const uint64_t bd = smem_desc(base + kW + (k >> 2) * kBBlk + off, 16, 1024, kSw128);
          umma_ss(tmem + (uint32_t)(acc * 256), a, bd, kId, k > 0);
        }
        umma_commit(mbar(bars, M_CEMPTY0 + st));
        umma_commit(mbar(bars, M_ACCF0 + acc));
        // Last item of this head: W may be replaced once these MMAs are done.
        if (it + 1 == it1 || (it + 1) / p.n_tiles != bh) umma_commit(mbar(bars, M_WEMPTY));
      }
      if (!ok) {
        umma_commit(mbar(bars, M_DRAIN));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(mbar(bars, M_DRAIN), 0) && globaltimer_ns() - t0 < p.wait_limit_ns) {
        }
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    // Thread = key row; TMEM lanes of warp w (w % 4 = lane quadrant) are rows 32 (w % 4) ...
    const int qd = warp & 3;
    for (int it = it0; it < it1; ++it) {
      const int i = it - it0, acc = i & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(mbar(bars, M_ACCF0 + acc), (i >> 1) & 1, ctl,
                                                        kDevTimeoutSoftmax));
      if (!ok) break;
      tc_fence_after();
      const int bh = it / p.n_tiles, tile = it - bh * p.n_tiles;
      const int b = bh / p.heads, h = bh - b * p.heads;
      const uint32_t t_row = tmem + (uint32_t)(acc * 256) + ((uint32_t)(qd * 32) << 16);
      uint8_t* stg = smem + kStg + (warp - 2) * kStgWarp;  // this warp's staging rows
      const int64_t j0 = (int64_t)tile * 128 + qd * 32;   // first key row of this warp
      uint32_t v[32];
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {  // 32-column chunks: 0-3 are K_h, 4-7 are V_h
        tmem_ld32(t_row + 32 * c, v);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7]));
          *reinterpret_cast<uint4*>(stg + lane * kStgRow + (c & 1) * 64 + q4 * 16) = w;
        }
        if (c & 1) {  // a 64-column block of 32 rows is staged: write it as whole lines
          __syncwarp();
          const int head = c < 4 ? h : p.heads + h;
          const int col0 = ((c >> 1) & 1) * 64;  // 0 or 64 within the head's 128 values
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int idx = lane + 32 * m, row = idx >> 3, q = idx & 7;
            const int64_t jr = j0 + row;
            if (jr < p.n_kv) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + row * kStgRow + q * 16);
              *reinterpret_cast<uint4*>(p.kv + (((int64_t)b * p.n_kv + jr) * (2 * p.heads) + head) * kDh + col0 +
                                        q * 8) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(mbar(bars, M_ACCE0 + acc));  // accumulator `acc` may be overwritten
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
  const int n_tiles = (int)((n_kv + 127) / 128);
  const int64_t items = (int64_t)batch * heads * n_tiles;
  if (items > 0x7FFFFFFF) return cudaErrorInvalidValue;
  static int sms[64] = {0};
  if (!sms[dev] && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidDevice;
  MatParams p{kv, status, kWaitLimitNs, n_kv, heads, n_tiles, (int)items};
  const int grid = items < sms[dev] ? (int)items : sms[dev];  // one CTA per SM (shared memory, TMEM)
  k_materialize_kv<<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace vmla
