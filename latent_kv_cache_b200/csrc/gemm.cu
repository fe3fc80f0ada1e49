// bf16 GEMM on the tensor cores for the projections either side of the latent
// attention: C[M x N] = A[M x K] . B[N x K]^T (nn.Linear weights), fp32
// accumulation in TMEM, bf16 output.  The N columns come from two weight matrices
// (B0 rows [0, N0), B1 rows [N0, N0 + N1)) written to two outputs, so the query
// and rope-query projections share one pass over the hidden states:
//     q   = x . W_Q^T    [tokens, H*128]
//     q_r = x . W_QR^T   [tokens, H*32]   (RoPE3D is applied by the attention kernel)
// and the output projection is the one-matrix case  y = o . W_O^T.
//
// Design: a persistent kernel over clusters of two CTAs on a CTA pair
// (tcgen05 cta_group::2).  One pair computes a 256 x 256 tile: CTA r stages A rows
// [128r, 128r + 128) and B rows [128r, 128r + 128) of the tile, and the leader
// CTA's single MMA thread issues M = 256, N = 256 MMAs that read both CTAs' shared
// memory and leave rows [128r, 128r + 128) of the fp32 tile in CTA r's TMEM.
// Every CTA therefore loads (128 + 128) x 64 operands per 128 x 256 x 64 of MMA
// work, half the bytes per FLOP of a one-CTA 128 x 256 tile; on this part the
// one-CTA tile was bound by the L2 -> SM operand traffic.
// TMEM holds two 256-column accumulators, so the epilogue of one tile overlaps
// the main loop of the next.
//
// 192 threads per CTA: warp 0 TMA producer (6-stage ring of [A 128x64 | B 128x64]
// 128B-swizzled k blocks), warp 1 TMEM allocation (+ the MMA issue in the leader),
// warps 2-5 the epilogue (TMEM lane = output row; each 64-column block of a warp's
// 32 rows is staged in shared memory and stored as whole 128-byte lines).  No multicast anywhere: each
// CTA loads its own operands and the MMA completions are committed to each CTA's
// barrier separately.  Every wait is bounded (abort flag + device status word).
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {
namespace {

constexpr int kThreads = 192;
constexpr int kTileM = 256, kTileN = 256, kBK = 64;  // per CTA pair
constexpr int kHalf = 128;                           // rows of A and of B each CTA stages
constexpr int kStages = 6;
constexpr uint32_t kABytes = kHalf * kBK * 2;        // 16 KB
constexpr uint32_t kBBytes = kHalf * kBK * 2;        // 16 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;  // 32 KB
constexpr uint32_t kBarOff = kStages * kStageBytes;  // 196608
// Epilogue staging: per epilogue warp, 32 rows x 64 bf16 (128 B) padded to 144 B
// so that row-per-lane writes hit distinct banks.
constexpr uint32_t kStgRow = 144;
constexpr uint32_t kStgWarp = 32 * kStgRow;
constexpr uint32_t kStg = kBarOff + 256;
constexpr uint32_t kSmemBytes = kStg + 4 * kStgWarp + 1024;
constexpr uint32_t kTmemCols = 512;                  // two 256-column accumulators

enum {
  G_FULL0 = 0,                   // leader: both CTAs' operand bytes of a stage landed
  G_EMPTY0 = kStages,            // each CTA: the MMAs reading a stage are done
  G_ACCF0 = 2 * kStages,         // each CTA: accumulator a holds a finished tile (x2)
  G_ACCE0 = 2 * kStages + 2,     // leader: both CTAs' epilogues drained accumulator a (x2)
  G_DRAIN = 2 * kStages + 4,
  G_COUNT
};
static_assert(8 * G_COUNT + 8 <= 256, "barrier area");

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
  int tiles_m, tiles_n;
  int* status;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ uint32_t gbar(uint32_t base, int i) { return base + 8u * i; }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (barriers that receive the peer CTA's arrivals).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, const WaitCtl& ctl, int code) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*ctl.abort_flag) return false;
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      *ctl.abort_flag = 1;
      atomicCAS(ctl.status, 0, code);
      return false;
    }
  }
}
// 2-D tile load into this CTA's shared memory; the completed bytes are counted on
// `bar_cluster`, which may be the leader CTA's barrier (the cta_group::2 form).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar_cluster, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrive on one CTA's barrier once this thread's earlier pair MMAs have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Tile schedule shared by the three roles.  Tiles whose N extent is full come
// first, then the last N column when it is partial (it issues narrower MMAs and
// costs less); tile positions are dealt to the pairs in rounds, alternating the
// direction every round, so that a pair that drew early in one round draws late
// in the next and the cheap partial tiles of the last rounds land on the pairs
// that have done the least.  Returns false once the pair has no i-th tile.
struct TileRef {
  int m0;      // first output row of the pair tile
  int n0;      // first output column
  int n;       // output columns of the tile (a multiple of 32, <= 256)
};
__device__ __forceinline__ bool tile_at(const GemmParams& p, int pair, int n_pairs, int i, TileRef& t) {
  const int pos = i * n_pairs + ((i & 1) ? n_pairs - 1 - pair : pair);
  const int n_tiles = p.tiles_m * p.tiles_n;
  if (pos >= n_tiles) return false;
  const int n_total = p.n0 + p.n1;
  const int full_n = n_total / kTileN;  // N tiles of the full width
  int mt, nt;
  if (pos < p.tiles_m * full_n) {
    mt = pos / full_n;
    nt = pos - mt * full_n;
  } else {  // the partial last column (tiles_n == full_n + 1)
    mt = pos - p.tiles_m * full_n;
    nt = full_n;
  }
  t.m0 = mt * kTileM;
  t.n0 = nt * kTileN;
  t.n = min(kTileN, n_total - t.n0);
  // Each CTA stages its n/2 B rows with one box from B0 or from B1: if N0 falls
  // inside one CTA's half, run the tile at full width instead (rows past N0 + N1
  // are zero-filled and their columns are not stored).
  if (t.n < kTileN && t.n0 < p.n0 && p.n0 < t.n0 + t.n && p.n0 != t.n0 + t.n / 2) t.n = kTileN;
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_bf16_pair(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~uintptr_t(1023)) - raw);  // kSmemBytes keeps 1 KB of slack
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + kBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * G_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = leader (issues the MMAs)
  const int pair = (int)cluster_id_x(), n_pairs = (int)cluster_count_x();
  const int nk = p.k / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(gbar(bars, G_FULL0 + s), 1);
      mbar_init(gbar(bars, G_EMPTY0 + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(gbar(bars, G_ACCF0 + a), 1);
      mbar_init(gbar(bars, G_ACCE0 + a), 8);  // 4 epilogue warps in each of the two CTAs
    }
    mbar_init(gbar(bars, G_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&maps.a);
      tma_prefetch_desc(&maps.b0);
      tma_prefetch_desc(&maps.b1);
      int last_use[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_use[s] = -1;
      int g = 0;
      bool ok = true;
      TileRef tr;
      for (int i = 0; ok && tile_at(p, pair, n_pairs, i, tr); ++i) {
        const int m0 = tr.m0 + kHalf * (int)rank;
        // B rows of the pair MMA are split in halves of tr.n / 2: CTA r stages rows
        // [r n/2, r n/2 + n/2) of the tile (the box always moves 128 rows; rows past
        // the half are not read, rows past the matrix are zero-filled).
        const int nrow = tr.n0 + (tr.n / 2) * (int)rank;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int st = g % kStages, use = g / kStages;
          if (use > 0 && !(ok = mbar_wait(gbar(bars, G_EMPTY0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer)))
            break;
          const uint32_t sa = base + st * kStageBytes;
          const uint32_t fb = map_to_rank(gbar(bars, G_FULL0 + st), 0);
          if (rank == 0) mbar_arrive_expect_tx(gbar(bars, G_FULL0 + st), 2 * kStageBytes);
          tma_load_2d_pair(sa, &maps.a, fb, kb * kBK, m0);
          if (nrow < p.n0) tma_load_2d_pair(sa + kABytes, &maps.b0, fb, kb * kBK, nrow);
          else tma_load_2d_pair(sa + kABytes, &maps.b1, fb, kb * kBK, nrow - p.n0);
          last_use[st] = use;
        }
      }
      if (!ok && rank == 0) {
        // Give in-flight loads (counted on the leader's barriers) time to land.
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
    if (lane == 0 && rank == 0) {
      const uint32_t peer = 1;
      int g = 0, i = 0;
      bool ok = true;
      TileRef tr;
      for (; ok && tile_at(p, pair, n_pairs, i, tr); ++i) {
        const uint32_t kId = idesc_bf16_f32(kTileM, tr.n, false, false);
        const int acc = i & 1, acc_use = i >> 1;
        if (acc_use > 0 &&
            !(ok = mbar_wait_cluster(gbar(bars, G_ACCE0 + acc), (acc_use - 1) & 1, ctl, kDevTimeoutMma)))
          break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * kTileN);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int st = g % kStages;
          if (!(ok = mbar_wait(gbar(bars, G_FULL0 + st), (g / kStages) & 1, ctl, kDevTimeoutMma))) break;
          tc_fence_after();
          const uint32_t sa = base + st * kStageBytes;
          const uint64_t a0 = smem_desc(sa, 16, 1024, kSw128);
          const uint64_t b0 = smem_desc(sa + kABytes, 16, 1024, kSw128);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // +32 bytes = +2 in the descriptor's address field
            umma_ss_pair(d, a0 + 2u * k, b0 + 2u * k, kId, (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit_pair(gbar(bars, G_EMPTY0 + st));
          umma_commit_pair(map_to_rank(gbar(bars, G_EMPTY0 + st), peer));
        }
        if (!ok) break;
        umma_commit_pair(gbar(bars, G_ACCF0 + acc));
        umma_commit_pair(map_to_rank(gbar(bars, G_ACCF0 + acc), peer));
      }
      if (!ok) {
        umma_commit_pair(gbar(bars, G_DRAIN));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(gbar(bars, G_DRAIN), 0) && globaltimer_ns() - t0 < p.wait_limit_ns) {
        }
      }
    }
  } else {
    // Epilogue warps 2..5: TMEM lane quadrant = warp % 4, row = 32 * quadrant + lane.
    const int qd = warp & 3;
    TileRef tr;
    for (int i = 0; tile_at(p, pair, n_pairs, i, tr); ++i) {
      const int acc = i & 1, acc_use = i >> 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(gbar(bars, G_ACCF0 + acc), acc_use & 1, ctl,
                                                        kDevTimeoutSoftmax));
      if (!ok) break;
      tc_fence_after();
      const int row0 = tr.m0 + kHalf * (int)rank + qd * 32;  // this warp's first row
      const int ncol0 = tr.n0;
      const uint32_t t_row = tmem + (uint32_t)(acc * kTileN) + ((uint32_t)(qd * 32) << 16);
      uint8_t* stg = smem + kStg + (warp - 2) * kStgWarp;
      uint32_t v[32];
      const int n_c = tr.n / 32;
#pragma unroll 1
      for (int c = 0; c < n_c; ++c) {
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
        if ((c & 1) || c == n_c - 1) {  // 64 (or a last 32) columns of 32 rows staged: store whole lines
          __syncwarp();
          // A 64-column block never straddles N0 (a multiple of 128).  When the tile
          // has an odd number of 32-column groups it ends at N0 + N1, so the stale
          // second half of its last block fails the column check below.
          const int col = ncol0 + 64 * (c >> 1);
          uint16_t* base_ptr = col < p.n0 ? p.c0 + col : p.c1 + (col - p.n0);
          const int64_t ld = col < p.n0 ? p.ldc0 : p.ldc1;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int idx = lane + 32 * m, r = idx >> 3, q = idx & 7;
            if (row0 + r < p.m && col + 8 * q < p.n0 + p.n1) {  // N1 is a multiple of 32
              const uint4 val = *reinterpret_cast<const uint4*>(stg + r * kStgRow + q * 16);
              *reinterpret_cast<uint4*>(base_ptr + (int64_t)(row0 + r) * ld + 8 * q) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(gbar(bars, G_ACCE0 + acc), 0));  // `acc` may be reused
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its barriers or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
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
  static int max_pairs[64] = {0};
  *encode_failed = false;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  if (!attr_done[dev]) {  // co-resident CTA pairs (one CTA per SM: shared memory and TMEM)
    cudaError_t e = cudaFuncSetAttribute(k_gemm_bf16_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)(sms & ~1), 1, 1);
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, k_gemm_bf16_pair, &cfg);
    if (e != cudaSuccess) return e;
    max_pairs[dev] = clusters > 0 ? clusters : 1;
    attr_done[dev] = true;
  }
  GemmMaps maps;
  bool ok = encode_rows(&maps.a, a, m, k) && encode_rows(&maps.b0, b0, n0, k);
  ok = ok && (n1 > 0 ? encode_rows(&maps.b1, b1, n1, k) : encode_rows(&maps.b1, b0, n0, k));
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  const int tiles_m = (m + kTileM - 1) / kTileM;
  const int tiles_n = (n0 + n1 + kTileN - 1) / kTileN;
  GemmParams p{c0, n1 > 0 ? c1 : c0, ldc0, n1 > 0 ? ldc1 : ldc0, m, n0, n1, k, tiles_m, tiles_n, status,
               kWaitLimitNs};
  const int64_t tiles = (int64_t)tiles_m * tiles_n;
  const int pairs = tiles < max_pairs[dev] ? (int)tiles : max_pairs[dev];
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_gemm_bf16_pair, maps, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace vmla
