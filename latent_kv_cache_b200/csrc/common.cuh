// Definitions shared by the kernels and the C-ABI layer of the library.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace vmla {

constexpr int kDc = 192;             // content latent width d_c
constexpr int kDr = 32;              // rope key width d_r
constexpr int kDrow = kDc + kDr;     // cached scalars per token (224)
constexpr int kDh = 128;             // per-head dim
constexpr int kPairsT = 6, kPairsH = 5, kPairsW = 5;  // rope split t:12 / h:10 / w:10 dims
constexpr int kMaxFrames = 32;       // frames spanned by one call
constexpr int kMaxSide = 256;        // max grid_h, grid_w
constexpr double kRopeTheta = 1.0e4;

// cos/sin of every rotary angle a call can need, passed by value as a kernel
// parameter (about 22 KB).  Entry [f][i] of `t` is frame t0 + f, pair i of the
// t axis; `h` and `w` are indexed by the row / column of the patch.
struct RopeTable {
  float2 t[kMaxFrames][kPairsT];
  float2 h[kMaxSide][kPairsH];
  float2 w[kMaxSide][kPairsW];
};

// What a host-side RopeTable currently holds (so that a call site can keep one
// table and refill only the parts whose positions changed).
struct RopeTableKey {
  int64_t t0 = -1;
  int n_frames = 0;
  int grid_h = 0, grid_w = 0;
};

// Host: make `tab` hold frames [t0, t0 + n_frames), rows [0, grid_h), cols [0, grid_w).
// Angles are computed in fp64 (pos * theta^(-2 i / d_axis)), then cos/sin in fp64
// and rounded to fp32.  `key` records what the table holds; entries that already
// hold the requested positions are not recomputed (a chunk's layers and denoising
// steps share t0 and the grid, and a rollout keeps its grid).
void build_rope_table(RopeTable* tab, RopeTableKey* key, int64_t t0, int n_frames, int grid_h, int grid_w);

// Work split of the latent attention launch: units (sample, query tile, head)
// [0, n_full) run whole, one CTA each; the tail_units after them run as `split`
// CTAs each over consecutive key ranges, merged by the part that finishes last
// (split == 1: no split).
struct SplitPlan {
  int64_t n_full;
  int split;
  int64_t tail_units;
};
constexpr int kMaxSplit = 8;
constexpr int kMinPartTiles = 32;  // key tiles of 128 keys per part, at least
SplitPlan plan_split(int64_t units, int n_kv_tiles, int sms);
int64_t split_workspace_bytes(const SplitPlan& plan, int d_c);
int sm_count_current_device();  // 0 when no device is current

// Device-side status word of the current device (lazily looked up, cached per device).
int* device_status_word();

// Per-wait limit used by all kernels (nanoseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace vmla
