/*
 * Reference (oracle) for the latent-cache append of VideoMLA.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code with the CUDA library.
 *
 * What it computes (VideoMLA, "Low-Rank Latent KV Cache for Minute-Scale
 * Autoregressive Video Diffusion": abstract; page "Approach"): every cached
 * video token stores a head-shared content latent c = x . W_DKV^T (d_c values)
 * and a head-shared decoupled positional key k_r = RoPE3D(x . W_KR^T) (d_r
 * values), 224 scalars in all.
 *
 * The order of the fp32 arithmetic is fixed here, so that a GPU kernel that
 * follows the same order reproduces it bit for bit:
 *   1. acc = 0; for k = 0 .. D-1 in increasing order: acc = fl32(acc + x[k] * w[k]).
 *      bf16 x bf16 products have at most 16 significant bits, so the product
 *      itself is exact in fp32 and each step rounds once.
 *   2. For the d_r rope columns, pair p = (2p, 2p+1) = (a, b) is rotated by the
 *      angle of its axis:  a' = fl32(fl32(a*cos) - fl32(b*sin)),
 *                          b' = fl32(fl32(a*sin) + fl32(b*cos)),
 *      with cos, sin = fp32 roundings of the fp64 libm cos/sin of the fp64 angle.
 *   3. Round to bf16, nearest, ties to even.
 * Rotary frequencies (reading of the pages, which give no formula): the 32 rope
 * dims split into (t: 12, h: 10, w: 10) blocks, pairs are adjacent dims inside
 * a block, and pair i of an axis with d_a dims turns at theta^(-2 i / d_a)
 * radians per position, theta = 1e4.  Positions of token n of a chunk that
 * starts at frame t0 on a grid_h x grid_w patch grid:
 *   t = t0 + n / (grid_h * grid_w),  row = (n / grid_w) % grid_h,  col = n % grid_w.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 * -ffp-contract=off keeps the rope products and sums as separate roundings.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* bf16 bits -> fp32, exact. */
static float bf16_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16 bits, round to nearest, ties to even (finite inputs). */
static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Rotary angle of pair `pair` (0 .. d_r/2 - 1) for position (t, row, col).
 * Axis blocks follow `split` = {d_t, d_h, d_w} dims. */
static double rope_angle(int pair, int64_t t, int64_t row, int64_t col,
                         const int split[3], double theta) {
    int p = pair;
    int axis = 0;
    while (axis < 3 && p >= split[axis] / 2) {
        p -= split[axis] / 2;
        axis++;
    }
    int64_t pos = axis == 0 ? t : (axis == 1 ? row : col);
    double freq = pow(theta, -2.0 * (double)p / (double)split[axis]);
    return (double)pos * freq;
}

/* fp32 cos/sin used by the append: fp32 rounding of fp64 libm values. */
void oracle_rope_cos_sin(int pair, int64_t t, int64_t row, int64_t col,
                         const int split[3], double theta, float* c, float* s) {
    double a = rope_angle(pair, t, row, col, split, theta);
    *c = (float)cos(a);
    *s = (float)sin(a);
}

/*
 * Ordered-fp32 append of n_tok tokens of B samples.
 *   x      [B, n_tok, D]           bf16 bits
 *   w_dkv  [d_c, D], w_kr [d_r, D] bf16 bits (nn.Linear layout [out, in])
 *   out32  [B, n_tok, d_c + d_r]   fp32 before the bf16 rounding (may be NULL)
 *   out    [B, n_tok, d_c + d_r]   bf16 bits (the cache rows)
 */
void oracle_cache_append(const uint16_t* x, const uint16_t* w_dkv, const uint16_t* w_kr,
                         int B, int n_tok, int D, int d_c, int d_r,
                         int64_t t0, int grid_h, int grid_w,
                         const int split[3], double theta,
                         float* out32, uint16_t* out) {
    const int width = d_c + d_r;
    const int64_t total = (int64_t)B * n_tok;
#pragma omp parallel for schedule(static)
    for (int64_t bn = 0; bn < total; ++bn) {
        const int64_t n = bn % n_tok;
        const uint16_t* xr = x + bn * D;
        float row_vals[1024];
        for (int j = 0; j < width; ++j) {
            const uint16_t* wr = j < d_c ? (w_dkv + (int64_t)j * D) : (w_kr + (int64_t)(j - d_c) * D);
            float acc = 0.0f;
            for (int k = 0; k < D; ++k) {
                float prod = bf16_to_float(xr[k]) * bf16_to_float(wr[k]);
                acc = acc + prod;
            }
            row_vals[j] = acc;
        }
        const int64_t per_frame = (int64_t)grid_h * grid_w;
        const int64_t t = t0 + n / per_frame;
        const int64_t row = (n / grid_w) % grid_h;
        const int64_t col = n % grid_w;
        for (int p = 0; p < d_r / 2; ++p) {
            float c, s;
            oracle_rope_cos_sin(p, t, row, col, split, theta, &c, &s);
            float a = row_vals[d_c + 2 * p];
            float b = row_vals[d_c + 2 * p + 1];
            float ac = a * c;
            float bs = b * s;
            float as = a * s;
            float bc = b * c;
            row_vals[d_c + 2 * p] = ac - bs;
            row_vals[d_c + 2 * p + 1] = as + bc;
        }
        for (int j = 0; j < width; ++j) {
            if (out32) out32[bn * width + j] = row_vals[j];
            out[bn * width + j] = float_to_bf16_rne(row_vals[j]);
        }
    }
}

/* Plain fp32 sequential dot product of bf16 vectors (exposed for the order pin). */
float oracle_ordered_dot(const uint16_t* a, const uint16_t* b, int n) {
    float acc = 0.0f;
    for (int k = 0; k < n; ++k) acc = acc + bf16_to_float(a[k]) * bf16_to_float(b[k]);
    return acc;
}

/* fp32 -> bf16 (RNE) of an array (exposed so tests can pin it to torch's cast). */
void oracle_round_bf16(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = float_to_bf16_rne(in[i]);
}
