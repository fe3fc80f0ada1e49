// Chunk attention over the latent KV cache (and the dense per-head baseline)
// on the sm_100a tensor cores.
//
// VideoMLA ("Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
// Diffusion", abstract; summary "Approach"): keys and values of every head are
// generated from one head-shared content latent c (d_c = 192 in the paper's
// model) plus one head-shared rope key k_r (32).  With W_UK absorbed into the query,
//     score(i, j) = scale * ( (q_h,i W_UK_h) . c_j + RoPE(q_r,h,i) . k_r,j ),
//     out_h,i     = ( sum_j softmax_j(score) c_j ) W_UV_h^T,
// so one CTA streams (d_c + 32)-wide cache rows [c ; k_r] and never materialises K or V.
//
// One CTA = one 128-query tile of one head of one sample; in the latent kernel heads
// are the fastest grid index so the 12 CTAs that read the same cache tiles run
// together and share them through L2 (the per-head dense and materialised kernels,
// further below, put query tiles fastest instead).  Warp roles (320 threads):
//   warp 0      TMA producer: prologue operands, then key tiles into a ring.
//   warp 1      TMEM allocation and the single MMA-issuing thread.
//   warps 2..9  two softmax warpgroups; in the latent kernel a thread owns one
//               query row (= TMEM lane) and one half of the columns of every
//               score tile (the per-head kernels give each warpgroup whole rows
//               of every other key tile instead).
//
// The latent kernel is a template over the content width d_c (64, 128, 192 or
// 256; the rope key stays 32 wide).  Its query operand Qa = [q_abs ; RoPE(q_r)]
// (128 x (d_c + 32) bf16) sits in shared memory, laid out like a key tile.
// MLA tensor memory (512 columns x 128 lanes, fp32 cells):
//   [0, d_c)    O_lat accumulator (the prologue's q_abs lands here first)
//   [256, 384)  S buffer 0 (P, bf16, overwrites its first 64 cells)
//   [384, 512)  S buffer 1
//   epilogue: normalised O_lat (bf16, d_c/2 cells) at 256, out accumulator at 384.
// Per 128-key tile j the MMA thread issues S_j = Qa K_j^T (d_c/16 + 2 MMAs,
// K = 16 each, the last two over the 64-byte-swizzled rope block) and then
// O += P_{j-1} C_{j-1} (8 MMAs of N = d_c, P read from TMEM, C read MN-major from
// the same shared-memory tile that served as K: keys and values are one tile).
// The softmax keeps the running max in log2 units and rescales O only when the
// max grows by more than 8 (P stays <= 2^8 in bf16).
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100.cuh"

namespace vmla {
namespace {

constexpr int kSoftmaxWarps = 8;                  // two warpgroups, one per half of a key tile
constexpr int kThreads = 64 + 32 * kSoftmaxWarps; // + producer warp + MMA warp
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kBM = 128;                          // queries per tile
constexpr uint32_t kTmemCols = 512;

// Per-head kernels (two-slot, below): the dense baseline (kKindDense) and attention
// over per-head keys/values materialised from the latent cache (kKindMat: content
// keys and values from a [B, n_kv, 2H, 128] buffer, the rope key straight from the
// latent cache).
enum Kind : int { kKindDense = 1, kKindMat = 2 };

// MLA: the Qa operand (128 x (d_c + 32) bf16) sits in shared memory (SS MMAs for
// the scores): O (d_c) + two 128-key S buffers (256) + Qa in TMEM would exceed
// the 512 TMEM columns, and 128-key score tiles matter more than the A source
// (a K = 16 tcgen05.mma takes at least ~93 cycles, so narrower N loses).
// The ring is as deep as shared memory allows: 6, 4, 3, 2 stages.
template <int kDcT>
struct Cfg {
  static_assert(kDcT == 64 || kDcT == 128 || kDcT == 192 || kDcT == 256, "d_c");
  static constexpr int kNb = kDcT / 64;                          // 128B-swizzled content blocks
  static constexpr int kBN = 128;                                // keys per tile
  static constexpr int kStages = kDcT == 64 ? 6 : kDcT == 128 ? 4 : kDcT == 192 ? 3 : 2;
  static constexpr uint32_t kBlkRows = 128 * 128;                // one 128B-swizzled block of a key tile
  static constexpr uint32_t kStage = kNb * kBlkRows + 128 * 64;  // [c: kNb blocks | k_r: 128 x 64 B]
  static constexpr uint32_t kQaBytes = kStage;                   // Qa tile, same block structure
  static constexpr int kOCols = kDcT;
  static constexpr uint32_t kTmemS0 = 256, kTmemS1 = 384;
  // With only two stages (d_c = 256) each stage is filled and released in three
  // parts with their own barriers: R = the rope block (free once the tile's scores
  // are done), X = content blocks [0, d_c/128) and Y = the other content blocks.
  // P.C runs as two N = d_c/2 halves, X is refilled while the second half runs,
  // and the next score tile takes its K steps in the order R, X, Y.
  static constexpr int kParts = kStages == 2 ? 3 : 1;
  static constexpr int kNbX = kParts == 3 ? kNb / 2 : kNb;  // content blocks in part X
};

constexpr uint32_t kBlk128 = 128 * 128;  // 128 rows x 128 B: prologue / epilogue operand blocks
constexpr uint32_t kTmemO = 0;

template <int kDcT>
struct Layout {
  using C = Cfg<kDcT>;
  static constexpr uint32_t kRingOff = C::kQaBytes;
  static constexpr uint32_t kBarOff = kRingOff + C::kStages * C::kStage;
  static constexpr uint32_t kRedOff = kBarOff + 512;
  static constexpr uint32_t kUsed = kRedOff + 2 * 2 * 128 * 4;
  static constexpr uint32_t kBytes = kUsed + 1024 <= 232448 ? kUsed + 1024 : 232448;
  static constexpr uint32_t kMaxPad = kBytes - kUsed;  // alignment slack the kernel checks for
  static_assert(kUsed + 512 <= 232448, "shared memory (with at least 512 B of alignment slack)");
  static_assert(C::kStages * C::kParts <= 8, "barrier slots");
};
// The MLA prologue parks q (2 blocks) and W_UK_h (d_c/64 blocks) in ring stages
// 0-1; the epilogue's W_UV_h (d_c/64 blocks) is one ring item.
template <int kDcT>
constexpr bool mla_fits() {
  using C = Cfg<kDcT>;
  return (2 + C::kNb) * kBlk128 <= 2 * C::kStage && C::kNb * kBlk128 <= C::kStage && C::kStages >= 2 &&
         kDcT + 256 <= (int)kTmemCols && kDcT / 2 <= 128;
}
static_assert(mla_fits<64>() && mla_fits<128>() && mla_fits<192>() && mla_fits<256>(), "MLA layout");

enum Bar {
  B_PRO = 0, B_QABS, B_QA,
  B_KVF0,                   // kStages "full" barriers per stage part
  B_KVE0 = B_KVF0 + 8,      // kStages "empty" barriers per stage part
  B_SF0 = B_KVE0 + 8, B_SF1,
  B_PF0, B_PF1,
  B_PV, B_OA, B_OUT, B_DRAIN,
  B_PART, B_LAST,           // split key range: partial written / last-part decision made
  B_MX0,                    // 8 barriers: (TMEM lane quadrant, tile parity)
  B_COUNT = B_MX0 + 8
};
static_assert(B_COUNT * 8 + 16 <= 512, "barrier area");

struct ChunkMaps {
  CUtensorMap q;    // [B, Nq, H, 128] box (64, 1, 128, 1), 128B swizzle
  CUtensorMap wuk;  // [H*128, d_c]         box (64, 128), 128B swizzle
  CUtensorMap wuv;  // [H*128, d_c]         box (64, 128), 128B swizzle
  CUtensorMap c;    // [B, n_kv, d_c + 32]  box (64, 128, 1), 128B swizzle (content latent)
  CUtensorMap kr;   // [B, n_kv, d_c + 32]  box (32, 128, 1), 64B swizzle (rope key, x = d_c)
};

struct AttnParams {
  const uint16_t* q;
  const uint16_t* q_rope;  // latent and materialised kernels
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
  // Latent kernel work split (1-D grid over units = (sample, query tile, head),
  // heads fastest).  Units [0, n_full) run whole, one CTA each.  Every later unit
  // runs as `split` CTAs over consecutive key-tile ranges; each writes its
  // unnormalised O_lat and its (running max, sum) to the workspace and counts
  // itself in; the part that arrives last merges all parts and runs the W_UV
  // epilogue.
  int n_full;
  int split;
  float* ws_o;    // [tail units * split][128][d_c] fp32
  float* ws_ml;   // [tail units * split][128][2] fp32: running max (log2 units), sum
  int* ws_cnt;    // [tail units] arrival counters, zero when the launch starts
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + 8u * i; }


// Maximum of three floats in one instruction (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
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

// Write one 16-byte chunk of row r into a 128B- / 64B-swizzled block (shared memory).
__device__ __forceinline__ void st_sw128_chunk(uint8_t* blk, int r, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(blk + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
}
__device__ __forceinline__ void st_sw64_chunk(uint8_t* blk, int r, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(blk + r * 64 + ((chunk ^ ((r >> 1) & 3)) << 4)) = v;
}

__device__ __forceinline__ uint32_t pack2(uint32_t lo, uint32_t hi, float scale) {
  return pack_bf16x2(__uint_as_float(lo) * scale, __uint_as_float(hi) * scale);
}
__device__ __forceinline__ uint4 pack8(const uint32_t* v, float scale) {
  return make_uint4(pack2(v[0], v[1], scale), pack2(v[2], v[3], scale), pack2(v[4], v[5], scale),
                    pack2(v[6], v[7], scale));
}

// Softmax roles: thread (half, quadrant qd, lane) owns query row r = 32 qd + lane,
// key columns [kBN/2 half, kBN/2 (half + 1)) of every S tile and output columns
// [half kOCols/2, (half + 1) kOCols/2).  The two halves of a row agree on the row
// maximum through `red` (shared memory, double-buffered by tile parity) and the
// barrier B_MX0 + 2 qd + parity (64 arrivals: the two warps of the quadrant).
struct SoftmaxThread {
  uint32_t t_row;  // TMEM address of lane r, column 0
  int half, qd, r;
  float* red;      // [2 parity][2 half][128 rows]
};

// Exchange a per-row value with the other half; returns the partner's value.
__device__ __forceinline__ bool exchange(const SoftmaxThread& t, uint32_t bars, int seq, float mine,
                                         float& theirs, const WaitCtl& ctl) {
  const int par = seq & 1;
  t.red[(par * 2 + t.half) * 128 + t.r] = mine;
  tc_fence_before();
  mbar_arrive(bar_addr(bars, B_MX0 + 2 * t.qd + par));
  if (!warp_wait(bar_addr(bars, B_MX0 + 2 * t.qd + par), (seq >> 1) & 1, ctl)) return false;
  tc_fence_after();
  theirs = t.red[(par * 2 + (t.half ^ 1)) * 128 + t.r];
  return true;
}

// Softmax step for key tile j.  Returns false on abort.
// j: tile index within this CTA's key range (barrier phases); jabs: the tile's
// index in the key sequence (masking of keys >= n_kv).
template <int kDcT>
__device__ __forceinline__ bool softmax_tile(int j, int jabs, uint32_t bars, const SoftmaxThread& t,
                                             const AttnParams& p, const WaitCtl& ctl,
                                             float& m_run, float& l_part) {
  using C = Cfg<kDcT>;
  constexpr int kW = C::kBN / 2;  // score columns per thread
  const int sb = j & 1;
  if (!warp_wait(bar_addr(bars, B_SF0 + sb), (j >> 1) & 1, ctl)) return false;
  tc_fence_after();
  const uint32_t sbase = sb ? C::kTmemS1 : C::kTmemS0;
  static_assert(kW == 64, "64 score columns per thread");
  float s[kW];
  {
    uint32_t ra[32], rb[32];
    tmem_ld32(t.t_row + sbase + kW * t.half, ra);
    tmem_ld32(t.t_row + sbase + kW * t.half + 32, rb);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) s[e] = __uint_as_float(ra[e]);
#pragma unroll
    for (int e = 0; e < kW - 32; ++e) s[32 + e] = __uint_as_float(rb[e]);
  }
  const int64_t kv0 = (int64_t)jabs * C::kBN + kW * t.half;
  if (kv0 + kW > p.n_kv) {
    const int64_t valid = p.n_kv - kv0;  // may be <= 0: the whole half is padding
#pragma unroll
    for (int c = 0; c < kW; ++c)
      if (c >= valid) s[c] = -INFINITY;
  }
  float mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mx[c] = max3f(s[c], s[8 + c], s[16 + c]);
#pragma unroll
  for (int c = 24; c < 56; c += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e) mx[e] = max3f(mx[e], s[c + e], s[c + 8 + e]);
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], s[56 + e]);
  mx[0] = max3f(mx[0], mx[1], mx[2]); mx[3] = max3f(mx[3], mx[4], mx[5]);
  mx[6] = fmaxf(mx[6], mx[7]);
  const float lmax = max3f(mx[0], mx[3], mx[6]);
  // The partner's columns of S are read before either half writes P over them.
  float omax;
  if (!exchange(t, bars, j, lmax, omax, ctl)) return false;
  const float m_tile = fmaxf(lmax, omax) * p.scale_log2;
  const bool need = m_tile > m_run + 8.0f;
  const float m_new = need ? m_tile : m_run;
  const float alpha = fast_exp2(m_run - m_new);
  // Pairs of scores in packed fp32x2 instructions (scale-and-subtract, row-sum
  // accumulators): fewer issue slots for the softmax warps, which share their
  // schedulers with the MMA-issuing thread.  acc[q] holds the sums of columns
  // 2e and 2e + 1 with e = q mod 4, the grouping of eight scalar accumulators.
  float2 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.0f, 0.0f);
  const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-m_new, -m_new);
  uint32_t pk[kW / 2];
#pragma unroll
  for (int e = 0; e < kW / 2; ++e) {
    const float2 x = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
    const float2 y = make_float2(fast_exp2(x.x), fast_exp2(x.y));
    acc[e & 3] = __fadd2_rn(acc[e & 3], y);
    pk[e] = pack_bf16x2(y.x, y.y);
  }
  // P (bf16 pairs) over the first kBN/2 cells of the S buffer: this half's kW/2 cells.
  tmem_st32(t.t_row + sbase + (kW / 2) * t.half, pk);
  acc[0] = __fadd2_rn(acc[0], acc[2]); acc[1] = __fadd2_rn(acc[1], acc[3]);
  acc[0] = __fadd2_rn(acc[0], acc[1]);
  l_part = l_part * alpha + (acc[0].x + acc[0].y);
  if (j > 0 && __any_sync(0xffffffffu, need)) {
    // O may only be rescaled once the previous P.C product has landed.  The PV
    // barrier cannot run ahead of PV(j-1) (PV(j) needs this tile's P), so its
    // parity identifies that phase even when earlier phases were not waited on.
    if (!warp_wait(bar_addr(bars, B_PV), (j - 1) & 1, ctl)) return false;
    tc_fence_after();
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < C::kOCols / 64; ++c) {
      const uint32_t col = kTmemO + t.half * (C::kOCols / 2) + 32 * c;
      tmem_ld32(t.t_row + col, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
      tmem_st32(t.t_row + col, r);
    }
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(bar_addr(bars, B_PF0 + sb));
  m_run = m_new;
  return true;
}

// Rope part of query qi of head h, rotated with the query's own (t, row, col);
// zeros for padding rows (qi >= n_q).
__device__ __forceinline__ void rope_query(const AttnParams& p, const RopeTable* tab, int b, int qi, int h,
                                           float (&qr)[kDr]) {
#pragma unroll
  for (int e = 0; e < kDr; ++e) qr[e] = 0.0f;
  if (qi >= p.n_q) return;
  const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDr);
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
    if (pr < kPairsT) cs = tab->t[f][pr];
    else if (pr < kPairsT + kPairsH) cs = tab->h[row][pr - kPairsT];
    else cs = tab->w[col][pr - kPairsT - kPairsH];
    const float a = qr[2 * pr], bb = qr[2 * pr + 1];
    qr[2 * pr] = a * cs.x - bb * cs.y;
    qr[2 * pr + 1] = a * cs.y + bb * cs.x;
  }
}

// ---------------------------------------------------------------------------
// The latent kernel: chunk attention with W_UK absorbed into the queries,
// [c ; k_r] key tiles that also serve as the values, and the W_UV epilogue, for
// content width kDcT.
// ---------------------------------------------------------------------------
template <int kDcT>
__device__ __forceinline__ void attn_body(const ChunkMaps& maps, const AttnParams& p, const RopeTable* tab) {
  using C = Cfg<kDcT>;
  using L = Layout<kDcT>;
  constexpr int kBN = C::kBN;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kStage = C::kStage;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uint32_t pad = (uint32_t)(((raw + 1023) & ~uintptr_t(1023)) - raw);
  if (pad > L::kMaxPad) {  // uniform across the CTA: nothing has started yet
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kDevSmemMisaligned);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t qa = smem_u32(smem);    // Qa tile (d_c/64 SW128 blocks + SW64 rope block)
  const uint32_t st0 = qa + L::kRingOff; // ring stage s at st0 + s * kStage
  const uint32_t bars = qa + L::kBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kBarOff + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_holder + 2);  // split: this part merges
  volatile int* skip_flag = reinterpret_cast<volatile int*>(tmem_holder + 3);  // split: no W_UV epilogue
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Grid order: heads fastest, so the 12 head-CTAs of a query tile, which read
  // the same cache tiles, run together.  1-D grid: whole units first, then the
  // parts of the split units.
  const int n_qt = (p.n_q + kBM - 1) / kBM;
  int unit = 0, part = 0, split = 1;
  {
    const int u = (int)blockIdx.x;
    if (u < p.n_full) {
      unit = u;
    } else {
      unit = p.n_full + (u - p.n_full) / p.split;
      part = (u - p.n_full) % p.split;
      split = p.split;
    }
  }
  const int per_b = n_qt * p.heads;
  const int b = unit / per_b;
  const int h = (unit % per_b) % p.heads;
  const int q0 = ((unit % per_b) / p.heads) * kBM;
  // This CTA's key tiles: [kt0, kt0 + n_tiles) of the n_kv_tiles tiles.
  const int kt0 = (int)((int64_t)part * p.n_kv_tiles / split);
  const int n_tiles = (int)((int64_t)(part + 1) * p.n_kv_tiles / split) - kt0;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, B_PRO), 1);
    mbar_init(bar_addr(bars, B_QABS), 1);
    mbar_init(bar_addr(bars, B_QA), kSoftmaxThreads);
    for (int s = 0; s < kStages * C::kParts; ++s) {  // part x of stage st: slot x * kStages + st
      mbar_init(bar_addr(bars, B_KVF0 + s), 1);
      mbar_init(bar_addr(bars, B_KVE0 + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_addr(bars, B_SF0 + s), 1);
      mbar_init(bar_addr(bars, B_PF0 + s), kSoftmaxThreads);
    }
    mbar_init(bar_addr(bars, B_PV), 1);
    mbar_init(bar_addr(bars, B_OA), kSoftmaxThreads);
    mbar_init(bar_addr(bars, B_OUT), 1);
    mbar_init(bar_addr(bars, B_DRAIN), 1);
    mbar_init(bar_addr(bars, B_PART), kSoftmaxThreads);
    mbar_init(bar_addr(bars, B_LAST), 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar_addr(bars, B_MX0 + i), 64);
    *abort_flag = 0;
    *last_flag = 0;
    *skip_flag = 0;
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
      constexpr int kParts = C::kParts;
      int last_use[kParts][kStages];
#pragma unroll
      for (int x = 0; x < kParts; ++x)
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_use[x][s] = -1;
      bool ok = true;
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.wuk);
      tma_prefetch_desc(&maps.wuv);
      tma_prefetch_desc(&maps.c);
      tma_prefetch_desc(&maps.kr);
      // Prologue operands borrow ring stages 0-1: q tile (2 blocks) then W_UK_h (d_c/64 blocks).
      mbar_arrive_expect_tx(bar_addr(bars, B_PRO), (2 + C::kNb) * kBlk128);
      tma_load_4d(st0, &maps.q, bar_addr(bars, B_PRO), 0, h, q0, b);
      tma_load_4d(st0 + kBlk128, &maps.q, bar_addr(bars, B_PRO), 64, h, q0, b);
#pragma unroll
      for (int i = 0; i < C::kNb; ++i)
        tma_load_2d(st0 + (2 + i) * kBlk128, &maps.wuk, bar_addr(bars, B_PRO), 64 * i, h * kDh);
      // n_tiles key tiles, then the W_UV_h blocks as one more ring item.
      const int n_items = n_tiles + 1;
      for (int i = 0; ok && i < n_items; ++i) {
        const int st = i % kStages, use = i / kStages;
        const uint32_t sa = st0 + st * kStage;
        if (use == 0 && st < 2) ok = mbar_wait(bar_addr(bars, B_QABS), 0, ctl, kDevTimeoutProducer);
        for (int x = 0; ok && x < kParts; ++x) {
          // Three-part stages: the W_UV item has no rope part (and is the stage's last use).
          if (kParts == 3 && x == 0 && i == n_tiles) continue;
          if (use > 0) ok = mbar_wait(bar_addr(bars, B_KVE0 + x * kStages + st), (use - 1) & 1, ctl,
                                      kDevTimeoutProducer);
          if (!ok) break;
          const uint32_t fb = bar_addr(bars, B_KVF0 + x * kStages + st);
          const int kv0 = (kt0 + i) * kBN;
          // part x: content blocks [blo, bhi) and (rope) the 64B-swizzled rope block
          const int blo = kParts == 1 ? 0 : x == 2 ? C::kNbX : 0;
          const int bhi = kParts == 1 ? C::kNb : x == 0 ? 0 : x == 1 ? C::kNbX : C::kNb;
          const bool rope = kParts == 1 || x == 0;
          if (i < n_tiles) {
            mbar_arrive_expect_tx(fb, (bhi - blo) * C::kBlkRows + (rope ? 128u * 64u : 0u));
            for (int blk = blo; blk < bhi; ++blk) tma_load_3d(sa + blk * C::kBlkRows, &maps.c, fb, 64 * blk, kv0, b);
            if (rope) tma_load_3d(sa + C::kNb * C::kBlkRows, &maps.kr, fb, kDcT, kv0, b);
          } else {
            mbar_arrive_expect_tx(fb, (bhi - blo) * kBlk128);
            for (int blk = blo; blk < bhi; ++blk) tma_load_2d(sa + blk * kBlk128, &maps.wuv, fb, 64 * blk, h * kDh);
          }
          last_use[x][st] = use;
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA exits.
        drain_wait(bar_addr(bars, B_PRO), 0, p.wait_limit_ns, p.status);
        for (int x = 0; x < kParts; ++x)
          for (int s = 0; s < kStages; ++s)
            if (last_use[x][s] >= 0)
              drain_wait(bar_addr(bars, B_KVF0 + x * kStages + s), last_use[x][s] & 1, p.wait_limit_ns, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------- MMA ----------------------------------
      constexpr uint32_t kIdS = idesc_bf16_f32(128, kBN, false, false);
      constexpr uint32_t kIdPv = idesc_bf16_f32(128, C::kOCols, false, true);
      bool ok = mbar_wait(bar_addr(bars, B_PRO), 0, ctl, kDevTimeoutMma);
      if (ok) {
        constexpr uint32_t kIdQabs = idesc_bf16_f32(128, kDcT, false, true);
        tc_fence_after();
        // q_abs = q_h . W_UK_h (M 128, N d_c, K 128): q K-major, W_UK MN-major.
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(st0 + (k >> 2) * kBlk128 + (k & 3) * 32, 16, 1024, kSw128);
          const uint64_t bd = smem_desc(st0 + 2 * kBlk128 + k * 2048, kBlk128, 1024, kSw128);
          umma_ss(tmem + kTmemO, a, bd, kIdQabs, k > 0);
        }
        umma_commit(bar_addr(bars, B_QABS));
      }
      if (ok) ok = mbar_wait(bar_addr(bars, B_QA), 0, ctl, kDevTimeoutMma);
      // The issuing thread shares its scheduler with two softmax warps, so it does
      // as little per MMA as it can: the descriptors of the Qa tile and of ring
      // stage 0 are built once, and a K step or another stage only moves the start
      // address (bits [0, 14), 16-byte units; every address here stays below
      // 2^18).  Ring positions advance as counters.
      const uint64_t dqa128 = smem_desc(qa, 16, 1024, kSw128), dqa64 = smem_desc(qa, 16, 512, kSw64);
      const uint64_t dst128 = smem_desc(st0, 16, 1024, kSw128), dst64 = smem_desc(st0, 16, 512, kSw64);
      const uint64_t dpv = smem_desc(st0, C::kBlkRows, 1024, kSw128);
      int pst = 0;  // ring stage of the tile whose P.C product is issued next
      auto issue_pv = [&](int jj) -> bool {
        if (!mbar_wait(bar_addr(bars, B_PF0 + (jj & 1)), (jj >> 1) & 1, ctl, kDevTimeoutMma))
          return false;
        tc_fence_after();
        // Value operand: the latent c blocks of the same stage, MN-major.
        const uint64_t dsv = dpv + pst * (kStage >> 4);
        const uint32_t a_t = tmem + ((jj & 1) ? C::kTmemS1 : C::kTmemS0);
        if constexpr (C::kParts == 3) {
          // Two halves of the latent columns; part X of the stage is free after the
          // first, part Y after the second.
          constexpr uint32_t kIdHalf = idesc_bf16_f32(128, 64 * C::kNbX, false, true);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int k = 0; k < kBN / 16; ++k)
              umma_ts(tmem + kTmemO + half * 64 * C::kNbX, a_t + k * 8,
                      dsv + ((half * C::kNbX * C::kBlkRows + k * 2048) >> 4), kIdHalf, (jj > 0 || k > 0) ? 1u : 0u);
            if (half == 0) umma_commit(bar_addr(bars, B_KVE0 + kStages + pst));
          }
          umma_commit(bar_addr(bars, B_PV));
          umma_commit(bar_addr(bars, B_KVE0 + 2 * kStages + pst));
        } else {
#pragma unroll
          for (int k = 0; k < kBN / 16; ++k)
            umma_ts(tmem + kTmemO, a_t + k * 8, dsv + ((k * 2048) >> 4), kIdPv, (jj > 0 || k > 0) ? 1u : 0u);
          umma_commit(bar_addr(bars, B_PV));
          umma_commit(bar_addr(bars, B_KVE0 + pst));
        }
        if (++pst == kStages) pst = 0;
        return true;
      };
      int st = 0, ph = 0;  // ring stage and phase of key tile j
      for (int j = 0; ok && j < n_tiles; ++j) {
        ok = mbar_wait(bar_addr(bars, B_KVF0 + st), ph, ctl, kDevTimeoutMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t so = st * (kStage >> 4);
        const uint32_t d = tmem + ((j & 1) ? C::kTmemS1 : C::kTmemS0);
        // S = Qa . [c ; k_r]^T (K = d_c + 32): d_c/16 steps over the 128B-swizzled
        // content blocks, 2 over the 64B-swizzled rope block; Qa and the key tile
        // share offsets.  With a stage in three parts the K steps run in the order
        // R (the rope block), X, Y, each part waited for just before its steps,
        // and R is released as soon as the scores are done.
        constexpr int kCs = 4 * C::kNb;
        constexpr int kCx = 4 * C::kNbX;  // content steps in part X
#pragma unroll
        for (int n = 0; n < kCs + 2; ++n) {
          const int k = C::kParts == 3 ? (n < 2 ? kCs + n : n - 2) : n;
          if (C::kParts == 3 && (n == 2 || n == 2 + kCx)) {  // (part R was waited for above)
            const int x = n == 2 ? 1 : 2;
            ok = mbar_wait(bar_addr(bars, B_KVF0 + x * kStages + st), ph, ctl, kDevTimeoutMma);
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t off =
              (k < kCs ? (k >> 2) * C::kBlkRows + (k & 3) * 32 : C::kNb * C::kBlkRows + (k - kCs) * 32) >> 4;
          umma_ss(d, (k < kCs ? dqa128 : dqa64) + off, (k < kCs ? dst128 : dst64) + so + off, kIdS, n > 0);
        }
        if (!ok) break;
        if constexpr (C::kParts == 3) umma_commit(bar_addr(bars, B_KVE0 + st));  // R free once S is done
        umma_commit(bar_addr(bars, B_SF0 + (j & 1)));
        if (j >= 1) ok = issue_pv(j - 1);
        if (++st == kStages) { st = 0; ph ^= 1; }
      }
      if (ok) ok = issue_pv(n_tiles - 1);
      if (ok) {
        constexpr uint32_t kIdOut = idesc_bf16_f32(128, 128, false, false);
        const int sw = n_tiles % kStages;
        // W_UV_h blocks: the whole stage, or parts X and Y of a three-part stage.
        const int ph = (n_tiles / kStages) & 1;
        ok = (C::kParts == 1
                  ? mbar_wait(bar_addr(bars, B_KVF0 + sw), ph, ctl, kDevTimeoutMma)
                  : mbar_wait(bar_addr(bars, B_KVF0 + kStages + sw), ph, ctl, kDevTimeoutMma) &&
                        mbar_wait(bar_addr(bars, B_KVF0 + 2 * kStages + sw), ph, ctl, kDevTimeoutMma)) &&
             mbar_wait(bar_addr(bars, B_OA), 0, ctl, kDevTimeoutMma);
        if (ok && !*skip_flag) {  // (a part of a split unit that does not merge skips it)
          tc_fence_after();
          const uint32_t wb = st0 + sw * kStage;
          // out = O_lat/l . W_UV_h^T (M 128, N 128, K d_c): A from TMEM, W_UV K-major.
#pragma unroll
          for (int k = 0; k < kDcT / 16; ++k) {
            const uint64_t bd = smem_desc(wb + (k >> 2) * kBlk128 + (k & 3) * 32, 16, 1024, kSw128);
            umma_ts(tmem + C::kTmemS1, tmem + C::kTmemS0 + k * 8, bd, kIdOut, k > 0);
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
    SoftmaxThread t;
    t.qd = warp & 3;
    t.half = (warp - 2) >> 2;
    t.r = t.qd * 32 + lane;
    t.t_row = tmem + ((uint32_t)(t.qd * 32) << 16);
    t.red = red;
    const int qi = q0 + t.r;
    bool ok = warp_wait(bar_addr(bars, B_QABS), 0, ctl);
    if (ok) {
      tc_fence_after();
      // q_abs (fp32, TMEM) -> bf16 Qa tile in shared memory; this half: columns
      // [d_c/2 half, +d_c/2).
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < C::kNb; ++c) {
        const int col = (kDcT / 2) * t.half + 32 * c;
        tmem_ld32(t.t_row + kTmemO + col, v);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          st_sw128_chunk(smem + (col >> 6) * C::kBlkRows, t.r, ((col & 63) >> 3) + q4, pack8(v + 8 * q4, 1.0f));
      }
      if (t.half == 0) {
        float qr[kDr];
        rope_query(p, tab, b, qi, h, qr);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 w;
          w.x = pack_bf16x2(qr[8 * c + 0], qr[8 * c + 1]);
          w.y = pack_bf16x2(qr[8 * c + 2], qr[8 * c + 3]);
          w.z = pack_bf16x2(qr[8 * c + 4], qr[8 * c + 5]);
          w.w = pack_bf16x2(qr[8 * c + 6], qr[8 * c + 7]);
          st_sw64_chunk(smem + C::kNb * C::kBlkRows, t.r, c, w);
        }
      }
      fence_proxy_async_smem();  // generic-proxy smem writes -> visible to the tensor core
    }
    if (ok) {
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(bars, B_QA));
    }
    float m_run = -INFINITY, l_part = 0.0f;
    for (int j = 0; ok && j < n_tiles; ++j)
      ok = softmax_tile<kDcT>(j, kt0 + j, bars, t, p, ctl, m_run, l_part);
    float l_other = 0.0f;
    if (ok) ok = exchange(t, bars, n_tiles, l_part, l_other, ctl);
    if (ok) ok = warp_wait(bar_addr(bars, B_PV), (n_tiles - 1) & 1, ctl);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / (l_part + l_other);
      uint16_t* out_row = p.out + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDh;
      uint32_t v[32];
      {
        // Split unit: write this part's partial, count it in, and find out whether
        // this part is the last of its unit (it then merges all parts).
        bool merge = false, emit = true;
        int slot0 = 0;
        // Partial O_lat layout: float4 (slot, half, 32-column group c, quarter q4,
        // row), so that each warp access is one contiguous 512 B run.
        auto part4 = [&](int slot, int c, int q4) -> float4* {
          return reinterpret_cast<float4*>(p.ws_o) + ((((int64_t)slot * 2 + t.half) * C::kNb + c) * 8 + q4) * kBM + t.r;
        };
        if (split > 1) {
          slot0 = (unit - p.n_full) * split;
#pragma unroll
          for (int c = 0; c < C::kNb; ++c) {  // this half's d_c/2 columns, 32 at a time
            tmem_ld32(t.t_row + kTmemO + (kDcT / 2) * t.half + 32 * c, v);
            tmem_ld_wait();
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *part4(slot0 + part, c, q4) = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                                        __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          }
          if (t.half == 0) {
            float2* ml = reinterpret_cast<float2*>(p.ws_ml) + (int64_t)(slot0 + part) * kBM + t.r;
            *ml = make_float2(m_run, l_part + l_other);
          }
          __threadfence();
          mbar_arrive(bar_addr(bars, B_PART));
          if (t.half == 0 && t.r == 0) {  // one thread counts the CTA in
            if (mbar_wait(bar_addr(bars, B_PART), 0, ctl, kDevTimeoutSoftmax)) {
              const int prev = atomicAdd(p.ws_cnt + (unit - p.n_full), 1);
              *last_flag = prev == split - 1 ? 1 : 0;
              mbar_arrive(bar_addr(bars, B_LAST));
            }
          }
          ok = warp_wait(bar_addr(bars, B_LAST), 0, ctl);
          merge = ok && *last_flag != 0;
          emit = merge;
          if (merge) __threadfence();
          if (!emit) *skip_flag = 1;
        }
        if (ok && emit) {
          // Normalised O_lat -> bf16 A operand of the W_UV MMA (this half: latent
          // [d_c/2 half, +d_c/2), i.e. d_c/4 cells).  Merging: the parts' O_lat
          // are brought to the common reference max and summed, over the summed l.
          const float2* ml = reinterpret_cast<const float2*>(p.ws_ml) + (int64_t)slot0 * kBM + t.r;
          float w_own = 1.0f, m_tot = m_run, scale_l = inv_l;
          if (merge) {
            for (int r2 = 0; r2 < split; ++r2)
              if (r2 != part) m_tot = fmaxf(m_tot, __ldcg(&ml[(int64_t)r2 * kBM].x));
            w_own = exp2f(m_run - m_tot);
            float l_tot = (l_part + l_other) * w_own;
            for (int r2 = 0; r2 < split; ++r2) {
              if (r2 == part) continue;
              const float2 mlr = __ldcg(&ml[(int64_t)r2 * kBM]);
              l_tot += mlr.y * exp2f(mlr.x - m_tot);
            }
            scale_l = 1.0f / l_tot;
          }
#pragma unroll
          for (int c = 0; c < C::kNb; ++c) {
            tmem_ld32(t.t_row + kTmemO + (kDcT / 2) * t.half + 32 * c, v);
            tmem_ld_wait();
            if (merge) {
              float acc[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(v[e]) * w_own;
              for (int r2 = 0; r2 < split; ++r2) {
                if (r2 == part) continue;
                const float w2 = exp2f(__ldcg(&ml[(int64_t)r2 * kBM].x) - m_tot);
                float4 fs[8];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) fs[q4] = __ldcg(part4(slot0 + r2, c, q4));
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                  const float4 f = fs[q4];
                  acc[4 * q4] = fmaf(f.x, w2, acc[4 * q4]);
                  acc[4 * q4 + 1] = fmaf(f.y, w2, acc[4 * q4 + 1]);
                  acc[4 * q4 + 2] = fmaf(f.z, w2, acc[4 * q4 + 2]);
                  acc[4 * q4 + 3] = fmaf(f.w, w2, acc[4 * q4 + 3]);
                }
              }
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(acc[e]);
            }
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack2(v[2 * e], v[2 * e + 1], scale_l);
            tmem_st16(t.t_row + C::kTmemS0 + (kDcT / 4) * t.half + 16 * c, pk);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(bar_addr(bars, B_OA));  // (a part that does not merge only releases the MMA thread)
        if (ok && emit) ok = warp_wait(bar_addr(bars, B_OUT), 0, ctl);
        if (ok && emit) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tmem_ld32(t.t_row + C::kTmemS1 + 64 * t.half + 32 * c, v);
            tmem_ld_wait();
            if (qi < p.n_q) {
              uint4* dst = reinterpret_cast<uint4*>(out_row + 64 * t.half + 32 * c);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) dst[q4] = pack8(v + 8 * q4, 1.0f);
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

template <int kDcT>
__global__ void __launch_bounds__(kThreads, 1)
    k_chunk_attn(const __grid_constant__ ChunkMaps maps, const __grid_constant__ AttnParams p,
                 const __grid_constant__ RopeTable tab) {
  attn_body<kDcT>(maps, p, &tab);
}

// ---------------------------------------------------------------------------
// Two-slot kernels for the per-head attention (dense baseline and materialised
// keys/values).  One CTA is one 128-query tile of one head of one sample, and
// its two softmax warpgroups do not split each score tile by columns as the
// latent kernel's do: warpgroup w ("slot" w) owns whole rows of every other key tile (tiles
// j = w, w + 2, ...), with its own score buffer S_w, its own output accumulator
// O_w and its own running max and sum; the two partial results are merged once,
// after the last tile.  So no per-tile exchange of row maxima is needed, and
// while one slot runs the exponentials of its tile the tensor pipe computes the
// other slot's scores and P.V products.  The query tile sits in shared memory
// (SS score MMAs), since tensor memory is taken up by the two S buffers and the
// two accumulators:
//   [0, 128) S_0 (P_0 as bf16 pairs over its first 64 cells)   [128, 256) S_1
//   [256, 384) O_0                                              [384, 512) O_1
// The MMA thread issues, after S_0(0) and S_1(1):
//   PV_0(0), S_0(2), PV_1(1), S_1(3), PV_0(2), S_0(4), ...
// so each slot's next score tile is queued right behind its own P.V product and
// a slot has the other slot's two MMA groups of time for its softmax.
// Key tiles (and the materialised variant's rope keys) and value tiles stream
// through two rings: a key stage is released when its scores are done, a value
// stage when its P.V product is.
// ---------------------------------------------------------------------------
template <int kKind>
struct HeadCfg {
  static constexpr bool kMat = kKind == kKindMat;
  static constexpr int kKSteps = kMat ? 10 : 8;                          // score K steps of 16
  static constexpr uint32_t kQBytes = 2 * kBlk128 + (kMat ? 128u * 64u : 0u);  // q_h (+ rope block)
  static constexpr uint32_t kKStage = kQBytes;                           // key tile: same block structure
  static constexpr uint32_t kVStage = 2 * kBlk128;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = kMat ? 2 : 3;
  static constexpr uint32_t kKOff = kQBytes;
  static constexpr uint32_t kVOff = kKOff + kKStages * kKStage;
  static constexpr uint32_t kBarOff = kVOff + kVStages * kVStage;
  static constexpr uint32_t kRedOff = kBarOff + 512;
  static constexpr uint32_t kUsed = kRedOff + 2 * 2 * 128 * 4;           // (m, l) of both slots
  static constexpr uint32_t kBytes = kUsed + 1024 <= 232448 ? kUsed + 1024 : 232448;
  static constexpr uint32_t kMaxPad = kBytes - kUsed;
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO0 = 256, kTmemO1 = 384;
  static_assert(kUsed + 512 <= 232448, "shared memory (with at least 512 B of alignment slack)");
};

enum HeadBar {
  P_Q = 0, P_QR,
  P_KF0, P_KE0 = P_KF0 + 3, P_VF0 = P_KE0 + 3, P_VE0 = P_VF0 + 3,
  P_SF0 = P_VE0 + 3, P_SF1, P_PF0, P_PF1, P_PV0, P_PV1,
  P_MRG, P_DRAIN,
  P_COUNT
};
static_assert(P_COUNT * 8 + 16 <= 512, "barrier area");

struct HeadMaps {
  CUtensorMap q;   // [B, Nq, H, 128] box (64, 1, 128, 1), 128B swizzle
  CUtensorMap k;   // dense: [B, Nk, H, 128]; materialised: [B, n_kv, 2H, 128] (keys at heads [0, H))
  CUtensorMap v;   // dense: [B, Nk, H, 128]; materialised: same tensor (values at head H + h)
  CUtensorMap kr;  // materialised only: latent cache [B, n_kv, 224] box (32, 128, 1), 64B swizzle
};

template <int kKind>
__device__ __forceinline__ void head_body(const HeadMaps& maps, const AttnParams& p, const RopeTable* tab) {
  using C = HeadCfg<kKind>;
  constexpr bool kMat = C::kMat;
  constexpr int kKS = C::kKStages, kVS = C::kVStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uint32_t pad = (uint32_t)(((raw + 1023) & ~uintptr_t(1023)) - raw);
  if (pad > C::kMaxPad) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kDevSmemMisaligned);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t qs = smem_u32(smem);  // query tile
  const uint32_t ks0 = qs + C::kKOff;  // key stage s at ks0 + s * kKStage
  const uint32_t vs0 = qs + C::kVOff;  // value stage s at vs0 + s * kVStage
  const uint32_t bars = qs + C::kBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * P_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);  // [slot][m | l][128 rows]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt = (p.n_q + kBM - 1) / kBM;
  const int h = (int)(blockIdx.x / n_qt);  // query tiles fastest: co-running CTAs share a head's K/V
  const int q0 = (int)(blockIdx.x % n_qt) * kBM;
  const int b = (int)blockIdx.y;
  const int n_tiles = p.n_kv_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, P_Q), 1);
    mbar_init(bar_addr(bars, P_QR), 128);
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar_addr(bars, P_KF0 + s), 1);
      mbar_init(bar_addr(bars, P_KE0 + s), 1);
      mbar_init(bar_addr(bars, P_VF0 + s), 1);
      mbar_init(bar_addr(bars, P_VE0 + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_addr(bars, P_SF0 + s), 1);
      mbar_init(bar_addr(bars, P_PF0 + s), 128);
      mbar_init(bar_addr(bars, P_PV0 + s), 1);
    }
    mbar_init(bar_addr(bars, P_MRG), kSoftmaxThreads);
    mbar_init(bar_addr(bars, P_DRAIN), 1);
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
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      if constexpr (kMat) tma_prefetch_desc(&maps.kr);
      mbar_arrive_expect_tx(bar_addr(bars, P_Q), 2 * kBlk128);
      tma_load_4d(qs, &maps.q, bar_addr(bars, P_Q), 0, h, q0, b);
      tma_load_4d(qs + kBlk128, &maps.q, bar_addr(bars, P_Q), 64, h, q0, b);
      int k_last[kKS], v_last[kVS];
#pragma unroll
      for (int s = 0; s < kKS; ++s) k_last[s] = -1;
#pragma unroll
      for (int s = 0; s < kVS; ++s) v_last[s] = -1;
      auto load_k = [&](int j) -> bool {
        const int st = j % kKS, use = j / kKS;
        if (use > 0 && !mbar_wait(bar_addr(bars, P_KE0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer))
          return false;
        const uint32_t fb = bar_addr(bars, P_KF0 + st), sa = ks0 + st * C::kKStage;
        const int kv0 = j * 128;
        mbar_arrive_expect_tx(fb, C::kKStage);
        tma_load_4d(sa, &maps.k, fb, 0, h, kv0, b);
        tma_load_4d(sa + kBlk128, &maps.k, fb, 64, h, kv0, b);
        if constexpr (kMat) tma_load_3d(sa + 2 * kBlk128, &maps.kr, fb, kDc, kv0, b);
        k_last[st] = use;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j % kVS, use = j / kVS;
        if (use > 0 && !mbar_wait(bar_addr(bars, P_VE0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer))
          return false;
        const uint32_t fb = bar_addr(bars, P_VF0 + st), sa = vs0 + st * C::kVStage;
        const int kv0 = j * 128;
        const int hv = kMat ? p.heads + h : h;  // materialised values follow the H key heads
        mbar_arrive_expect_tx(fb, C::kVStage);
        tma_load_4d(sa, &maps.v, fb, 0, hv, kv0, b);
        tma_load_4d(sa + kBlk128, &maps.v, fb, 64, hv, kv0, b);
        v_last[st] = use;
        return true;
      };
      // In the order the MMA thread consumes them: K0, K1, then V_j, K_{j+2}.
      bool ok = load_k(0);
      if (ok && n_tiles > 1) ok = load_k(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        ok = load_v(j);
        if (ok && j + 2 < n_tiles) ok = load_k(j + 2);
      }
      if (!ok) {
        // Let every copy already issued land before the CTA exits.
        drain_wait(bar_addr(bars, P_Q), 0, p.wait_limit_ns, p.status);
        for (int s = 0; s < kKS; ++s)
          if (k_last[s] >= 0) drain_wait(bar_addr(bars, P_KF0 + s), k_last[s] & 1, p.wait_limit_ns, p.status);
        for (int s = 0; s < kVS; ++s)
          if (v_last[s] >= 0) drain_wait(bar_addr(bars, P_VF0 + s), v_last[s] & 1, p.wait_limit_ns, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------- MMA ----------------------------------
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPv = idesc_bf16_f32(128, kDh, false, true);
      bool ok = mbar_wait(bar_addr(bars, P_Q), 0, ctl, kDevTimeoutMma);
      if (ok && kMat) ok = mbar_wait(bar_addr(bars, P_QR), 0, ctl, kDevTimeoutMma);
      // The issuing thread shares its scheduler with two softmax warps, so it does
      // as little per MMA as it can: the descriptors of the query tile and of key
      // and value stage 0 are built once, and a K step or another stage only moves
      // the start address (bits [0, 14), 16-byte units; every address here stays
      // below 2^18).  Ring positions advance as counters.
      const uint64_t dq128 = smem_desc(qs, 16, 1024, kSw128), dq64 = smem_desc(qs, 16, 512, kSw64);
      const uint64_t dk128 = smem_desc(ks0, 16, 1024, kSw128), dk64 = smem_desc(ks0, 16, 512, kSw64);
      const uint64_t dv = smem_desc(vs0, kBlk128, 1024, kSw128);
      int kst = 0, kph = 0, vst = 0, vph = 0;
      // S_w = Q . K_j^T (w = j & 1) for the next key tile j: 8 steps over the
      // 128B-swizzled blocks (+2 over the 64B-swizzled rope block); the query and
      // key tiles share offsets.
      auto issue_s = [&](int w) -> bool {
        if (!mbar_wait(bar_addr(bars, P_KF0 + kst), kph, ctl, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t so = kst * (C::kKStage >> 4);
        const uint32_t d = tmem + (w ? C::kTmemS1 : C::kTmemS0);
#pragma unroll
        for (int k = 0; k < C::kKSteps; ++k) {
          const uint32_t off = (k < 8 ? (k >> 2) * kBlk128 + (k & 3) * 32 : 2 * kBlk128 + (k - 8) * 32) >> 4;
          umma_ss(d, (k < 8 ? dq128 : dq64) + off, (k < 8 ? dk128 : dk64) + so + off, kIdS, k > 0);
        }
        umma_commit(bar_addr(bars, P_SF0 + w));
        umma_commit(bar_addr(bars, P_KE0 + kst));
        if (++kst == kKS) { kst = 0; kph ^= 1; }
        return true;
      };
      // O_w += P_w . V_j: P from TMEM (bf16 pairs over S_w), V MN-major.
      auto issue_pv = [&](int j) -> bool {
        const int w = j & 1;
        if (!mbar_wait(bar_addr(bars, P_PF0 + w), (j >> 1) & 1, ctl, kDevTimeoutMma)) return false;
        if (!mbar_wait(bar_addr(bars, P_VF0 + vst), vph, ctl, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint64_t dvs = dv + vst * (C::kVStage >> 4);
        const uint32_t a_t = tmem + (w ? C::kTmemS1 : C::kTmemS0);
        const uint32_t d = tmem + (w ? C::kTmemO1 : C::kTmemO0);
#pragma unroll
        for (int k = 0; k < 8; ++k) umma_ts(d, a_t + k * 8, dvs + k * (2048 >> 4), kIdPv, (j >= 2 || k > 0) ? 1u : 0u);
        umma_commit(bar_addr(bars, P_PV0 + w));
        umma_commit(bar_addr(bars, P_VE0 + vst));
        if (++vst == kVS) { vst = 0; vph ^= 1; }
        return true;
      };
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
      if (ok && n_tiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        ok = issue_pv(j);
        if (ok && j + 2 < n_tiles) ok = issue_s(j & 1);  // tile j + 2, same slot as j
      }
      if (!ok) {
        umma_commit(bar_addr(bars, P_DRAIN));
        drain_wait(bar_addr(bars, P_DRAIN), 0, p.wait_limit_ns, p.status);
      }
    }
  } else {
    // -------------------------------- softmax ---------------------------------
    const int qd = warp & 3;
    const int slot = (warp - 2) >> 2;
    const int r = qd * 32 + lane;
    const uint32_t t_row = tmem + ((uint32_t)(qd * 32) << 16);
    const uint32_t s_col = slot ? C::kTmemS1 : C::kTmemS0;
    const uint32_t o_col = slot ? C::kTmemO1 : C::kTmemO0;
    const int qi = q0 + r;
    bool ok = true;
    if constexpr (kMat) {
      if (slot == 0) {  // rope block of the query tile: RoPE(q_r) of this row
        float qr[kDr];
        rope_query(p, tab, b, qi, h, qr);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 w4;
          w4.x = pack_bf16x2(qr[8 * c + 0], qr[8 * c + 1]);
          w4.y = pack_bf16x2(qr[8 * c + 2], qr[8 * c + 3]);
          w4.z = pack_bf16x2(qr[8 * c + 4], qr[8 * c + 5]);
          w4.w = pack_bf16x2(qr[8 * c + 6], qr[8 * c + 7]);
          st_sw64_chunk(smem + 2 * kBlk128, r, c, w4);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_addr(bars, P_QR));
      }
    }
    const int n_mine = (n_tiles - slot + 1) / 2;  // tiles slot, slot + 2, ...
    float m_run = -INFINITY, l_run = 0.0f;
    for (int i = 0; ok && i < n_mine; ++i) {
      const int j = 2 * i + slot;
      if (!warp_wait(bar_addr(bars, P_SF0 + slot), i & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      float s[128];
      {
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_row + s_col + 32 * c, sr + 32 * c);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(sr[e]);
      }
      const int64_t kv0 = (int64_t)j * 128;
      if (kv0 + 128 > p.n_kv) {
        const int64_t valid = p.n_kv - kv0;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx[c] = s[c];
#pragma unroll
      for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      mx[0] = fmaxf(mx[0], mx[4]); mx[1] = fmaxf(mx[1], mx[5]);
      mx[2] = fmaxf(mx[2], mx[6]); mx[3] = fmaxf(mx[3], mx[7]);
      mx[0] = fmaxf(mx[0], mx[2]); mx[1] = fmaxf(mx[1], mx[3]);
      const float m_tile = fmaxf(mx[0], mx[1]) * p.scale_log2;
      const bool need = m_tile > m_run + 8.0f;
      const float m_new = need ? m_tile : m_run;
      const float alpha = fast_exp2(m_run - m_new);
      float sum[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) sum[c] = 0.0f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = fast_exp2(fmaf(s[64 * c + 2 * e], p.scale_log2, -m_new));
          const float p1 = fast_exp2(fmaf(s[64 * c + 2 * e + 1], p.scale_log2, -m_new));
          sum[(2 * e) & 7] += p0;
          sum[(2 * e + 1) & 7] += p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(t_row + s_col + 32 * c, pk);  // P over the first 64 cells of S_w
      }
      sum[0] += sum[4]; sum[1] += sum[5]; sum[2] += sum[6]; sum[3] += sum[7];
      sum[0] += sum[2]; sum[1] += sum[3];
      l_run = l_run * alpha + (sum[0] + sum[1]);
      if (i > 0 && __any_sync(0xffffffffu, need)) {
        // O_w is rescaled once this slot's previous P.V product has landed (its
        // next one waits for this tile's P, so the barrier is not ahead of it).
        if (!warp_wait(bar_addr(bars, P_PV0 + slot), (i - 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t o[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(t_row + o_col + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_row + o_col + 32 * c, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(bars, P_PF0 + slot));
      m_run = m_new;
    }
    // Merge: both slots' last P.V products have landed; each slot writes half of
    // the output columns from both accumulators.
    if (ok && n_mine > 0) ok = warp_wait(bar_addr(bars, P_PV0 + slot), (n_mine - 1) & 1, ctl);
    red[(slot * 2 + 0) * 128 + r] = m_run;
    red[(slot * 2 + 1) * 128 + r] = l_run;
    tc_fence_before();
    mbar_arrive(bar_addr(bars, P_MRG));
    if (ok) ok = warp_wait(bar_addr(bars, P_MRG), 0, ctl);
    if (ok) {
      tc_fence_after();
      const bool two = n_tiles > 1;  // slot 1 had key tiles (else O_1 was never written)
      const float m0 = red[r], l0 = red[128 + r];
      const float m1 = two ? red[256 + r] : -INFINITY, l1 = two ? red[384 + r] : 0.0f;
      const float m = fmaxf(m0, m1);
      const float a0 = fast_exp2(m0 - m);
      const float a1 = two ? fast_exp2(m1 - m) : 0.0f;
      const float inv_l = 1.0f / (a0 * l0 + a1 * l1);
      const float w0 = a0 * inv_l, w1 = a1 * inv_l;
      uint16_t* out_row = p.out + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDh;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = 64 * slot + 32 * c;
        uint32_t v0[32], v1[32];
        tmem_ld32(t_row + C::kTmemO0 + col, v0);
        if (two) tmem_ld32(t_row + C::kTmemO1 + col, v1);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0 = __uint_as_float(v0[2 * e]) * w0, x1 = __uint_as_float(v0[2 * e + 1]) * w0;
          if (two) {
            x0 = fmaf(__uint_as_float(v1[2 * e]), w1, x0);
            x1 = fmaf(__uint_as_float(v1[2 * e + 1]), w1, x1);
          }
          pk[e] = pack_bf16x2(x0, x1);
        }
        if (qi < p.n_q) {
          uint4* dst = reinterpret_cast<uint4*>(out_row + col);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
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

__global__ void __launch_bounds__(kThreads, 1)
    k_dense_attn(const __grid_constant__ HeadMaps maps, const __grid_constant__ AttnParams p) {
  head_body<kKindDense>(maps, p, nullptr);
}

__global__ void __launch_bounds__(kThreads, 1)
    k_mat_attn(const __grid_constant__ HeadMaps maps, const __grid_constant__ AttnParams p,
               const __grid_constant__ RopeTable tab) {
  head_body<kKindMat>(maps, p, &tab);
}

// ---------------------------------------------------------------------------
// Two-slot latent kernel for content widths d_c <= 128.  The latent kernel above
// splits every score tile by columns between its two softmax warpgroups; at
// d_c <= 128 tensor memory also holds two O_lat accumulators, so here, as in
// the per-head kernels, softmax warpgroup w owns whole rows of key tiles
// j = w, w + 2, ... with its own S buffer, O_lat accumulator, max and sum, and
// the two partial results are merged once before the W_UV epilogue.
//   [0, 128) S_0 / P_0    [128, 256) S_1 / P_1    [256, 256 + d_c) O_0
//   [384, 384 + d_c) O_1 (q_abs lands in O_0 first)
//   epilogue: merged O_lat / l in bf16 at 0 (d_c/2 cells), out accumulator at 128.
// Keys and values are one ring of [c ; k_r] tiles; a stage is released once its
// tile's P.C product is done.  The units are those of the latent kernel (heads
// fastest), without key-range parts.
// ---------------------------------------------------------------------------
template <int kDcT>
struct SlotCfg {
  static_assert(kDcT == 64 || kDcT == 128, "two-slot latent kernel: d_c 64 or 128");
  static constexpr int kNb = kDcT / 64;                          // 128B-swizzled content blocks
  static constexpr uint32_t kStage = kNb * kBlk128 + 128 * 64;   // [c: kNb blocks | k_r: 128 x 64 B]
  static constexpr int kStages = kDcT == 64 ? 8 : 4;
  static constexpr int kCs = 4 * kNb;                            // content K steps of the scores
  static constexpr uint32_t kRingOff = kStage;                   // after the Qa tile
  static constexpr uint32_t kBarOff = kRingOff + kStages * kStage;
  static constexpr uint32_t kRedOff = kBarOff + 512;
  static constexpr uint32_t kUsed = kRedOff + 2 * 2 * 128 * 4;   // (m, l) of both slots
  static constexpr uint32_t kBytes = kUsed + 1024 <= 232448 ? kUsed + 1024 : 232448;
  static constexpr uint32_t kMaxPad = kBytes - kUsed;
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO0 = 256, kTmemO1 = 384;
  static_assert(kUsed + 512 <= 232448, "shared memory (with at least 512 B of alignment slack)");
  // The prologue parks the q tile (2 blocks) and W_UK_h (kNb blocks) in ring stages 0-1.
  static_assert((2 + kNb) * kBlk128 <= 2 * kStage && kNb * kBlk128 <= kStage, "prologue operands");
};

enum SlotBar {
  L_PRO = 0, L_QABS, L_QA,
  L_F0, L_E0 = L_F0 + 8,
  L_SF0 = L_E0 + 8, L_SF1, L_PF0, L_PF1, L_PV0, L_PV1,
  L_MRG, L_OA, L_OUT, L_DRAIN,
  L_COUNT
};
static_assert(L_COUNT * 8 + 16 <= 512, "barrier area");

template <int kDcT>
__device__ __forceinline__ void slot_body(const ChunkMaps& maps, const AttnParams& p, const RopeTable* tab) {
  using C = SlotCfg<kDcT>;
  constexpr int kS = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uint32_t pad = (uint32_t)(((raw + 1023) & ~uintptr_t(1023)) - raw);
  if (pad > C::kMaxPad) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kDevSmemMisaligned);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t qa = smem_u32(smem);      // Qa tile
  const uint32_t st0 = qa + C::kRingOff;   // ring stage s at st0 + s * kStage
  const uint32_t bars = qa + C::kBarOff;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * L_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);  // [slot][m | l][128 rows]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt = (p.n_q + kBM - 1) / kBM;
  const int unit = (int)blockIdx.x;
  const int per_b = n_qt * p.heads;
  const int b = unit / per_b;
  const int h = (unit % per_b) % p.heads;
  const int q0 = ((unit % per_b) / p.heads) * kBM;
  const int n_tiles = p.n_kv_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar_addr(bars, L_PRO), 1);
    mbar_init(bar_addr(bars, L_QABS), 1);
    mbar_init(bar_addr(bars, L_QA), kSoftmaxThreads);
    for (int s = 0; s < kS; ++s) {
      mbar_init(bar_addr(bars, L_F0 + s), 1);
      mbar_init(bar_addr(bars, L_E0 + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_addr(bars, L_SF0 + s), 1);
      mbar_init(bar_addr(bars, L_PF0 + s), 128);
      mbar_init(bar_addr(bars, L_PV0 + s), 1);
    }
    mbar_init(bar_addr(bars, L_MRG), kSoftmaxThreads);
    mbar_init(bar_addr(bars, L_OA), kSoftmaxThreads);
    mbar_init(bar_addr(bars, L_OUT), 1);
    mbar_init(bar_addr(bars, L_DRAIN), 1);
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
      int last_use[kS];
#pragma unroll
      for (int s = 0; s < kS; ++s) last_use[s] = -1;
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.wuk);
      tma_prefetch_desc(&maps.wuv);
      tma_prefetch_desc(&maps.c);
      tma_prefetch_desc(&maps.kr);
      mbar_arrive_expect_tx(bar_addr(bars, L_PRO), (2 + C::kNb) * kBlk128);
      tma_load_4d(st0, &maps.q, bar_addr(bars, L_PRO), 0, h, q0, b);
      tma_load_4d(st0 + kBlk128, &maps.q, bar_addr(bars, L_PRO), 64, h, q0, b);
#pragma unroll
      for (int i = 0; i < C::kNb; ++i)
        tma_load_2d(st0 + (2 + i) * kBlk128, &maps.wuk, bar_addr(bars, L_PRO), 64 * i, h * kDh);
      bool ok = true;
      int st = 0, use = 0;
      // n_tiles key tiles, then the W_UV_h blocks as one more ring item.
      for (int i = 0; ok && i <= n_tiles; ++i) {
        if (use == 0 && st < 2) ok = mbar_wait(bar_addr(bars, L_QABS), 0, ctl, kDevTimeoutProducer);
        if (ok && use > 0) ok = mbar_wait(bar_addr(bars, L_E0 + st), (use - 1) & 1, ctl, kDevTimeoutProducer);
        if (!ok) break;
        const uint32_t fb = bar_addr(bars, L_F0 + st), sa = st0 + st * C::kStage;
        if (i < n_tiles) {
          const int kv0 = i * 128;
          mbar_arrive_expect_tx(fb, C::kStage);
          for (int blk = 0; blk < C::kNb; ++blk) tma_load_3d(sa + blk * kBlk128, &maps.c, fb, 64 * blk, kv0, b);
          tma_load_3d(sa + C::kNb * kBlk128, &maps.kr, fb, kDcT, kv0, b);
        } else {
          mbar_arrive_expect_tx(fb, C::kNb * kBlk128);
          for (int blk = 0; blk < C::kNb; ++blk) tma_load_2d(sa + blk * kBlk128, &maps.wuv, fb, 64 * blk, h * kDh);
        }
        last_use[st] = use;
        if (++st == kS) { st = 0; ++use; }
      }
      if (!ok) {
        drain_wait(bar_addr(bars, L_PRO), 0, p.wait_limit_ns, p.status);
        for (int s = 0; s < kS; ++s)
          if (last_use[s] >= 0) drain_wait(bar_addr(bars, L_F0 + s), last_use[s] & 1, p.wait_limit_ns, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------- MMA ----------------------------------
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPv = idesc_bf16_f32(128, kDcT, false, true);
      bool ok = mbar_wait(bar_addr(bars, L_PRO), 0, ctl, kDevTimeoutMma);
      if (ok) {
        tc_fence_after();
        // q_abs = q_h . W_UK_h (M 128, N d_c, K 128) into O_0: q K-major, W_UK MN-major.
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(st0 + (k >> 2) * kBlk128 + (k & 3) * 32, 16, 1024, kSw128);
          const uint64_t bd = smem_desc(st0 + 2 * kBlk128 + k * 2048, kBlk128, 1024, kSw128);
          umma_ss(tmem + C::kTmemO0, a, bd, kIdPv, k > 0);
        }
        umma_commit(bar_addr(bars, L_QABS));
      }
      if (ok) ok = mbar_wait(bar_addr(bars, L_QA), 0, ctl, kDevTimeoutMma);
      // Descriptors built once; a K step or another stage only moves the start
      // address (bits [0, 14), 16-byte units; every address here is below 2^18).
      const uint64_t dqa128 = smem_desc(qa, 16, 1024, kSw128), dqa64 = smem_desc(qa, 16, 512, kSw64);
      const uint64_t dst128 = smem_desc(st0, 16, 1024, kSw128), dst64 = smem_desc(st0, 16, 512, kSw64);
      const uint64_t dpv = smem_desc(st0, kBlk128, 1024, kSw128);
      int sst = 0, sph = 0, pst = 0;  // ring positions of the next score tile and P.C product
      // S_w = Qa . [c ; k_r]^T for the next key tile (w = its parity).
      auto issue_s = [&](int w) -> bool {
        if (!mbar_wait(bar_addr(bars, L_F0 + sst), sph, ctl, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t so = sst * (C::kStage >> 4);
        const uint32_t d = tmem + (w ? C::kTmemS1 : C::kTmemS0);
#pragma unroll
        for (int k = 0; k < C::kCs + 2; ++k) {
          const uint32_t off = (k < C::kCs ? (k >> 2) * kBlk128 + (k & 3) * 32 : C::kNb * kBlk128 + (k - C::kCs) * 32) >> 4;
          umma_ss(d, (k < C::kCs ? dqa128 : dqa64) + off, (k < C::kCs ? dst128 : dst64) + so + off, kIdS, k > 0);
        }
        umma_commit(bar_addr(bars, L_SF0 + w));
        if (++sst == kS) { sst = 0; sph ^= 1; }
        return true;
      };
      // O_w += P_w . C_j: P from TMEM, the latent c blocks of tile j's stage MN-major.
      auto issue_pv = [&](int j) -> bool {
        const int w = j & 1;
        if (!mbar_wait(bar_addr(bars, L_PF0 + w), (j >> 1) & 1, ctl, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint64_t dsv = dpv + pst * (C::kStage >> 4);
        const uint32_t a_t = tmem + (w ? C::kTmemS1 : C::kTmemS0);
        const uint32_t d = tmem + (w ? C::kTmemO1 : C::kTmemO0);
#pragma unroll
        for (int k = 0; k < 8; ++k) umma_ts(d, a_t + k * 8, dsv + k * (2048 >> 4), kIdPv, (j >= 2 || k > 0) ? 1u : 0u);
        umma_commit(bar_addr(bars, L_PV0 + w));
        umma_commit(bar_addr(bars, L_E0 + pst));
        if (++pst == kS) pst = 0;
        return true;
      };
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
      if (ok && n_tiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        ok = issue_pv(j);
        if (ok && j + 2 < n_tiles) ok = issue_s(j & 1);  // tile j + 2, same slot as j
      }
      if (ok) {
        // out = O_lat/l . W_UV_h^T (M 128, N 128, K d_c): A from TMEM, W_UV K-major.
        const int sw = n_tiles % kS;
        ok = mbar_wait(bar_addr(bars, L_F0 + sw), (n_tiles / kS) & 1, ctl, kDevTimeoutMma) &&
             mbar_wait(bar_addr(bars, L_OA), 0, ctl, kDevTimeoutMma);
        if (ok) {
          tc_fence_after();
          constexpr uint32_t kIdOut = idesc_bf16_f32(128, 128, false, false);
          const uint32_t wb = st0 + sw * C::kStage;
#pragma unroll
          for (int k = 0; k < kDcT / 16; ++k) {
            const uint64_t bd = smem_desc(wb + (k >> 2) * kBlk128 + (k & 3) * 32, 16, 1024, kSw128);
            umma_ts(tmem + C::kTmemS1, tmem + C::kTmemS0 + k * 8, bd, kIdOut, k > 0);
          }
          umma_commit(bar_addr(bars, L_OUT));
        }
      }
      if (!ok) {
        umma_commit(bar_addr(bars, L_DRAIN));
        drain_wait(bar_addr(bars, L_DRAIN), 0, p.wait_limit_ns, p.status);
      }
    }
  } else {
    // -------------------------------- softmax ---------------------------------
    const int qd = warp & 3;
    const int slot = (warp - 2) >> 2;
    const int r = qd * 32 + lane;
    const uint32_t t_row = tmem + ((uint32_t)(qd * 32) << 16);
    const uint32_t s_col = slot ? C::kTmemS1 : C::kTmemS0;
    const uint32_t o_col = slot ? C::kTmemO1 : C::kTmemO0;
    const int qi = q0 + r;
    // q_abs (fp32, O_0) -> bf16 Qa tile in shared memory; this slot converts
    // latent columns [d_c/2 slot, +d_c/2), the first slot also the rope block.
    bool ok = warp_wait(bar_addr(bars, L_QABS), 0, ctl);
    if (ok) {
      tc_fence_after();
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < C::kNb; ++c) {
        const int col = (kDcT / 2) * slot + 32 * c;
        tmem_ld32(t_row + C::kTmemO0 + col, v);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          st_sw128_chunk(smem + (col >> 6) * kBlk128, r, ((col & 63) >> 3) + q4, pack8(v + 8 * q4, 1.0f));
      }
      if (slot == 0) {
        float qr[kDr];
        rope_query(p, tab, b, qi, h, qr);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 w4;
          w4.x = pack_bf16x2(qr[8 * c + 0], qr[8 * c + 1]);
          w4.y = pack_bf16x2(qr[8 * c + 2], qr[8 * c + 3]);
          w4.z = pack_bf16x2(qr[8 * c + 4], qr[8 * c + 5]);
          w4.w = pack_bf16x2(qr[8 * c + 6], qr[8 * c + 7]);
          st_sw64_chunk(smem + C::kNb * kBlk128, r, c, w4);
        }
      }
      fence_proxy_async_smem();  // generic-proxy smem writes -> visible to the tensor core
      tc_fence_before();
      mbar_arrive(bar_addr(bars, L_QA));
    }
    // The per-tile step is the per-head kernels' (written out again: as one shared
    // inline function it made ptxas spill and measured 0.5-1.8% slower).
    const int n_mine = (n_tiles - slot + 1) / 2;  // tiles slot, slot + 2, ...
    float m_run = -INFINITY, l_run = 0.0f;
    for (int i = 0; ok && i < n_mine; ++i) {
      const int j = 2 * i + slot;
      if (!warp_wait(bar_addr(bars, L_SF0 + slot), i & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      float s[128];
      {
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_row + s_col + 32 * c, sr + 32 * c);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(sr[e]);
      }
      const int64_t kv0 = (int64_t)j * 128;
      if (kv0 + 128 > p.n_kv) {
        const int64_t valid = p.n_kv - kv0;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx[c] = s[c];
#pragma unroll
      for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      mx[0] = fmaxf(mx[0], mx[4]); mx[1] = fmaxf(mx[1], mx[5]);
      mx[2] = fmaxf(mx[2], mx[6]); mx[3] = fmaxf(mx[3], mx[7]);
      mx[0] = fmaxf(mx[0], mx[2]); mx[1] = fmaxf(mx[1], mx[3]);
      const float m_tile = fmaxf(mx[0], mx[1]) * p.scale_log2;
      const bool need = m_tile > m_run + 8.0f;
      const float m_new = need ? m_tile : m_run;
      const float alpha = fast_exp2(m_run - m_new);
      float sum[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) sum[c] = 0.0f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = fast_exp2(fmaf(s[64 * c + 2 * e], p.scale_log2, -m_new));
          const float p1 = fast_exp2(fmaf(s[64 * c + 2 * e + 1], p.scale_log2, -m_new));
          sum[(2 * e) & 7] += p0;
          sum[(2 * e + 1) & 7] += p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(t_row + s_col + 32 * c, pk);  // P over the first 64 cells of S_w
      }
      sum[0] += sum[4]; sum[1] += sum[5]; sum[2] += sum[6]; sum[3] += sum[7];
      sum[0] += sum[2]; sum[1] += sum[3];
      l_run = l_run * alpha + (sum[0] + sum[1]);
      if (i > 0 && __any_sync(0xffffffffu, need)) {
        // O_w is rescaled once this slot's previous P.C product has landed (its
        // next one waits for this tile's P, so the barrier is not ahead of it).
        if (!warp_wait(bar_addr(bars, L_PV0 + slot), (i - 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t o[32];
#pragma unroll
        for (int c = 0; c < kDcT / 32; ++c) {
          tmem_ld32(t_row + o_col + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(t_row + o_col + 32 * c, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(bars, L_PF0 + slot));
      m_run = m_new;
    }
    // Merge: both slots' last P.C products have landed; each slot writes half of
    // the normalised O_lat (bf16, the A operand of the W_UV product) from both
    // accumulators.
    if (ok && n_mine > 0) ok = warp_wait(bar_addr(bars, L_PV0 + slot), (n_mine - 1) & 1, ctl);
    red[(slot * 2 + 0) * 128 + r] = m_run;
    red[(slot * 2 + 1) * 128 + r] = l_run;
    tc_fence_before();
    mbar_arrive(bar_addr(bars, L_MRG));
    if (ok) ok = warp_wait(bar_addr(bars, L_MRG), 0, ctl);
    if (ok) {
      tc_fence_after();
      const bool two = n_tiles > 1;  // slot 1 had key tiles (else O_1 was never written)
      const float m0 = red[r], l0 = red[128 + r];
      const float m1 = two ? red[256 + r] : -INFINITY, l1 = two ? red[384 + r] : 0.0f;
      const float m = fmaxf(m0, m1);
      const float a0 = fast_exp2(m0 - m);
      const float a1 = two ? fast_exp2(m1 - m) : 0.0f;
      const float inv_l = 1.0f / (a0 * l0 + a1 * l1);
      const float w0 = a0 * inv_l, w1 = a1 * inv_l;
#pragma unroll
      for (int c = 0; c < C::kNb; ++c) {
        const int col = (kDcT / 2) * slot + 32 * c;
        uint32_t v0[32], v1[32];
        tmem_ld32(t_row + C::kTmemO0 + col, v0);
        if (two) tmem_ld32(t_row + C::kTmemO1 + col, v1);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0 = __uint_as_float(v0[2 * e]) * w0, x1 = __uint_as_float(v0[2 * e + 1]) * w0;
          if (two) {
            x0 = fmaf(__uint_as_float(v1[2 * e]), w1, x0);
            x1 = fmaf(__uint_as_float(v1[2 * e + 1]), w1, x1);
          }
          pk[e] = pack_bf16x2(x0, x1);
        }
        tmem_st16(t_row + C::kTmemS0 + (kDcT / 4) * slot + 16 * c, pk);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    mbar_arrive(bar_addr(bars, L_OA));
    if (ok) ok = warp_wait(bar_addr(bars, L_OUT), 0, ctl);
    if (ok) {
      tc_fence_after();
      uint16_t* out_row = p.out + (((int64_t)b * p.n_q + qi) * p.heads + h) * kDh;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tmem_ld32(t_row + C::kTmemS1 + 64 * slot + 32 * c, v);
        tmem_ld_wait();
        if (qi < p.n_q) {
          uint4* dst = reinterpret_cast<uint4*>(out_row + 64 * slot + 32 * c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) dst[q4] = pack8(v + 8 * q4, 1.0f);
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

template <int kDcT>
__global__ void __launch_bounds__(kThreads, 1)
    k_chunk_attn_slots(const __grid_constant__ ChunkMaps maps, const __grid_constant__ AttnParams p,
                       const __grid_constant__ RopeTable tab) {
  slot_body<kDcT>(maps, p, &tab);
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

bool set_smem_attr(const void* fn, int bytes, bool* done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

// [B, rows, H, 128] bf16, box of 128 rows x 64 elements of one head.
bool make_head_map(CUtensorMap* m, const uint16_t* t, int batch, int64_t n_rows, int heads) {
  const cuuint64_t dims[4] = {(cuuint64_t)kDh, (cuuint64_t)heads, (cuuint64_t)n_rows, (cuuint64_t)batch};
  const cuuint64_t strides[3] = {(cuuint64_t)kDh * 2, (cuuint64_t)heads * kDh * 2,
                                 (cuuint64_t)n_rows * heads * kDh * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kBM, 1};
  return make_map(m, t, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

namespace {

// Workspace of the split key ranges, laid out [O partials | (m, l) | counters].
struct SplitLayout {
  int64_t o_bytes, ml_bytes, cnt_bytes, total;
};
SplitLayout split_layout(int64_t tail_units, int split, int d_c) {
  auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
  SplitLayout l;
  l.o_bytes = up(tail_units * split * kBM * d_c * 4);
  l.ml_bytes = up(tail_units * split * kBM * 8);
  l.cnt_bytes = up(tail_units * 4);
  l.total = l.o_bytes + l.ml_bytes + l.cnt_bytes;
  return l;
}

template <int kDcT>
cudaError_t launch_chunk_attention_t(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                     const uint16_t* w_uv, const uint16_t* cache, int batch, int n_q, int heads,
                                     int64_t cap, int64_t n_kv, int64_t t0, int grid_h, int grid_w, float scale,
                                     uint16_t* out, int* status, cudaStream_t stream, bool* encode_failed,
                                     const SplitPlan& plan, void* workspace) {
  using C = Cfg<kDcT>;
  using L = Layout<kDcT>;
  constexpr int kRow = kDcT + kDr;
  static bool attr_done[64] = {false};
  *encode_failed = false;
  // d_c <= 128 without key-range parts: the two-slot kernel (two O_lat fit in TMEM).
  constexpr bool kSlots = kDcT <= 128;
  if (kSlots && plan.split == 1) {
    if constexpr (kSlots) {
      static bool slot_attr_done[64] = {false};
      if (!set_smem_attr((const void*)k_chunk_attn_slots<kDcT>, SlotCfg<kDcT>::kBytes, slot_attr_done))
        return cudaErrorInvalidValue;
    }
  } else if (!set_smem_attr((const void*)k_chunk_attn<kDcT>, L::kBytes, attr_done)) {
    return cudaErrorInvalidValue;
  }
  ChunkMaps maps;
  bool ok = make_head_map(&maps.q, q, batch, n_q, heads);
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kDcT, (cuuint64_t)heads * kDh};
    const cuuint64_t strides[1] = {(cuuint64_t)kDcT * 2};
    const cuuint32_t box[2] = {64, 128};
    ok = ok && make_map(&maps.wuk, w_uk, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&maps.wuv, w_uv, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kRow, (cuuint64_t)n_kv, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)kRow * 2, (cuuint64_t)cap * kRow * 2};
    const cuuint32_t box_c[3] = {64, (cuuint32_t)C::kBN, 1};
    const cuuint32_t box_r[3] = {32, (cuuint32_t)C::kBN, 1};
    ok = ok && make_map(&maps.c, cache, 3, dims, strides, box_c, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&maps.kr, cache, 3, dims, strides, box_r, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnParams p{};
  p.q = q;
  p.q_rope = q_rope;
  p.out = out;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  p.n_kv = n_kv;
  p.n_q = n_q;
  p.heads = heads;
  p.n_kv_tiles = (int)((n_kv + C::kBN - 1) / C::kBN);
  p.grid_h = grid_h;
  p.grid_w = grid_w;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.n_full = (int)plan.n_full;
  p.split = plan.split;
  int64_t blocks = plan.n_full;
  if (plan.split > 1) {
    const SplitLayout sl = split_layout(plan.tail_units, plan.split, kDcT);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.ws_o = reinterpret_cast<float*>(ws);
    p.ws_ml = reinterpret_cast<float*>(ws + sl.o_bytes);
    p.ws_cnt = reinterpret_cast<int*>(ws + sl.o_bytes + sl.ml_bytes);
    cudaError_t e = cudaMemsetAsync(p.ws_cnt, 0, plan.tail_units * sizeof(int), stream);
    if (e != cudaSuccess) return e;
    blocks += plan.tail_units * plan.split;
  }
  static thread_local RopeTable tab;
  static thread_local RopeTableKey tab_key;
  const int per_frame = grid_h * grid_w;
  build_rope_table(&tab, &tab_key, t0, (n_q + per_frame - 1) / per_frame, grid_h, grid_w);
  if constexpr (kSlots) {
    if (plan.split == 1) {
      k_chunk_attn_slots<kDcT><<<dim3((unsigned)blocks), kThreads, SlotCfg<kDcT>::kBytes, stream>>>(maps, p, tab);
      return cudaGetLastError();
    }
  }
  k_chunk_attn<kDcT><<<dim3((unsigned)blocks), kThreads, L::kBytes, stream>>>(maps, p, tab);
  return cudaGetLastError();
}

}  // namespace

int sm_count_current_device() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = sms;
  }
  return cached[dev];
}

// One latent-attention CTA per SM at a time (shared memory and TMEM).  Units
// (sample, query tile, head) fill whole waves of `sms`; when the last wave is
// partial, its units may run as `split` parts over key ranges so that the tail
// takes ceil(split * rem / sms) / split of a whole unit's time instead of one.
// Every part repeats the unit's prologue (query tile, q.W_UK) and adds its
// partial's write, the count-in and the last part's merge, so a part keeps at
// least kMinPartTiles key tiles: measured on the small workload (5 key tiles,
// 24 units) a 5-way split took 2.5x the unsplit launch, while at 1080P (574 key
// tiles, 84 tail units, 7-way) it saved 1.5% in an interleaved A/B.
SplitPlan plan_split(int64_t units, int n_kv_tiles, int sms) {
  SplitPlan s{units, 1, 0};
  if (sms <= 0 || units <= 0) return s;
  const int64_t full = units / sms * sms, rem = units - full;
  if (rem == 0) return s;
  double best = 1.0;
  for (int k = 2; k <= kMaxSplit && k * kMinPartTiles <= n_kv_tiles; ++k) {
    const double tail = (double)((k * rem + sms - 1) / sms) / k;
    if (tail < best - 1e-9) {
      best = tail;
      s.split = k;
    }
  }
  if (s.split > 1) {
    s.n_full = full;
    s.tail_units = rem;
  }
  return s;
}

int64_t split_workspace_bytes(const SplitPlan& plan, int d_c) {
  return plan.split > 1 ? split_layout(plan.tail_units, plan.split, d_c).total : 0;
}

// d_c in {64, 128, 192, 256}; the caller has validated it.  `plan` says which
// units run whole; with plan.split > 1, `workspace` holds split_workspace_bytes.
cudaError_t launch_chunk_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* w_uk,
                                   const uint16_t* w_uv, const uint16_t* cache, int batch, int n_q,
                                   int heads, int d_c, int64_t cap, int64_t n_kv, int64_t t0, int grid_h,
                                   int grid_w, float scale, uint16_t* out, int* status,
                                   cudaStream_t stream, bool* encode_failed, const SplitPlan& plan,
                                   void* workspace) {
  switch (d_c) {
    case 64:
      return launch_chunk_attention_t<64>(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                          grid_w, scale, out, status, stream, encode_failed, plan, workspace);
    case 128:
      return launch_chunk_attention_t<128>(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                           grid_w, scale, out, status, stream, encode_failed, plan, workspace);
    case 192:
      return launch_chunk_attention_t<192>(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                           grid_w, scale, out, status, stream, encode_failed, plan, workspace);
    case 256:
      return launch_chunk_attention_t<256>(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, cap, n_kv, t0, grid_h,
                                           grid_w, scale, out, status, stream, encode_failed, plan, workspace);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dense_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int batch,
                                   int n_q, int64_t n_kv, int heads, float scale, uint16_t* out,
                                   int* status, cudaStream_t stream, bool* encode_failed) {
  static bool attr_done[64] = {false};
  *encode_failed = false;
  if (!set_smem_attr((const void*)k_dense_attn, HeadCfg<kKindDense>::kBytes, attr_done)) return cudaErrorInvalidValue;
  HeadMaps maps;
  bool ok = make_head_map(&maps.q, q, batch, n_q, heads) && make_head_map(&maps.k, k, batch, n_kv, heads) &&
            make_head_map(&maps.v, v, batch, n_kv, heads);
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnParams p{};
  p.q = q;
  p.out = out;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  p.n_kv = n_kv;
  p.n_q = n_q;
  p.heads = heads;
  p.n_kv_tiles = (int)((n_kv + 127) / 128);
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  dim3 grid((unsigned)(((n_q + kBM - 1) / kBM) * heads), (unsigned)batch);
  k_dense_attn<<<grid, kThreads, HeadCfg<kKindDense>::kBytes, stream>>>(maps, p);
  return cudaGetLastError();
}

cudaError_t launch_mat_attention(const uint16_t* q, const uint16_t* q_rope, const uint16_t* kv,
                                 const uint16_t* cache, int batch, int n_q, int heads, int64_t cap,
                                 int64_t n_kv, int64_t t0, int grid_h, int grid_w, float scale, uint16_t* out,
                                 int* status, cudaStream_t stream, bool* encode_failed) {
  static bool attr_done[64] = {false};
  *encode_failed = false;
  if (!set_smem_attr((const void*)k_mat_attn, HeadCfg<kKindMat>::kBytes, attr_done)) return cudaErrorInvalidValue;
  HeadMaps maps;
  bool ok = make_head_map(&maps.q, q, batch, n_q, heads) && make_head_map(&maps.k, kv, batch, n_kv, 2 * heads) &&
            make_head_map(&maps.v, kv, batch, n_kv, 2 * heads);
  {
    const cuuint64_t dims[3] = {(cuuint64_t)kDrow, (cuuint64_t)n_kv, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)kDrow * 2, (cuuint64_t)cap * kDrow * 2};
    const cuuint32_t box_r[3] = {32, 128, 1};
    ok = ok && make_map(&maps.kr, cache, 3, dims, strides, box_r, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!ok) {
    *encode_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnParams p{};
  p.q = q;
  p.q_rope = q_rope;
  p.out = out;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  p.n_kv = n_kv;
  p.n_q = n_q;
  p.heads = heads;
  p.n_kv_tiles = (int)((n_kv + 127) / 128);
  p.grid_h = grid_h;
  p.grid_w = grid_w;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  static thread_local RopeTable tab;
  static thread_local RopeTableKey tab_key;
  const int per_frame = grid_h * grid_w;
  build_rope_table(&tab, &tab_key, t0, (n_q + per_frame - 1) / per_frame, grid_h, grid_w);
  dim3 grid((unsigned)(((n_q + kBM - 1) / kBM) * heads), (unsigned)batch);
  k_mat_attn<<<grid, kThreads, HeadCfg<kKindMat>::kBytes, stream>>>(maps, p, tab);
  return cudaGetLastError();
}

}  // namespace vmla
