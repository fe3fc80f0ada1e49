// Device status word, rope-table construction and the failure-path self-test.
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {

// One status word per device that loads the library (a few bytes, never freed).
__device__ int g_device_status[4];

int* device_status_word() {
  static std::mutex mu;
  static int* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<int*>(p);
  }
  return cached[dev];
}

void build_rope_table(RopeTable* tab, RopeTableKey* key, int64_t t0, int n_frames, int grid_h, int grid_w) {
  const int split[3] = {2 * kPairsT, 2 * kPairsH, 2 * kPairsW};
  n_frames = n_frames < kMaxFrames ? n_frames : kMaxFrames;
  grid_h = grid_h < kMaxSide ? grid_h : kMaxSide;
  grid_w = grid_w < kMaxSide ? grid_w : kMaxSide;
  if (key->t0 != t0 || key->n_frames < n_frames) {
    for (int f = 0; f < n_frames; ++f) {
      for (int i = 0; i < kPairsT; ++i) {
        double freq = std::pow(kRopeTheta, -2.0 * (double)i / (double)split[0]);
        double a = (double)(t0 + f) * freq;
        tab->t[f][i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    key->t0 = t0;
    key->n_frames = n_frames;
  }
  if (key->grid_h < grid_h) {  // rows [0, key->grid_h) already hold their values
    for (int r = key->grid_h; r < grid_h; ++r) {
      for (int i = 0; i < kPairsH; ++i) {
        double freq = std::pow(kRopeTheta, -2.0 * (double)i / (double)split[1]);
        double a = (double)r * freq;
        tab->h[r][i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    key->grid_h = grid_h;
  }
  if (key->grid_w < grid_w) {
    for (int c = key->grid_w; c < grid_w; ++c) {
      for (int i = 0; i < kPairsW; ++i) {
        double freq = std::pow(kRopeTheta, -2.0 * (double)i / (double)split[2]);
        double a = (double)c * freq;
        tab->w[c][i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    key->grid_w = grid_w;
  }
}

// Waits on a barrier that nothing completes; gives up after limit_ns.
__global__ void k_selftest_wait_timeout(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtl ctl{&abort_flag, status, limit_ns};
    mbar_wait(smem_u32(&bar), 0, ctl, kDevTimeoutSelftest);
  }
  __syncthreads();
}

cudaError_t launch_selftest_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t s) {
  k_selftest_wait_timeout<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace vmla
