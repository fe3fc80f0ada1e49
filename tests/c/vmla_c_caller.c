/*
 * A plain C caller of the library's C ABI (include/videomla.h), with no Python
 * and no PyTorch in the process: the CUDA runtime supplies device memory.
 *
 *   vmla_c_caller <dir>
 *
 * <dir>/meta.txt holds "batch n_q n_kv heads d_model chunk_t0 grid_h grid_w scale".
 * Inputs (bf16 bits, little-endian uint16, row-major): x.bin [B, n_kv, D] (every
 * frame of the window), w_dkv.bin [192, D], w_kr.bin [32, D], q.bin [B, n_q, H, 128],
 * q_rope.bin [B, n_q, H, 32], w_uk.bin / w_uv.bin [H*128, 192], k.bin / v.bin
 * [B, n_kv, H, 128].  The program appends the window one 3-frame chunk per call
 * (slots = token index), runs the latent chunk attention and the dense attention,
 * and writes cache.bin [B, n_kv, 224], out.bin and out_dense.bin [B, n_q, H, 128].
 * Exit status 0 on success; on a failed call it prints the library's message.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "videomla.h"

static void* read_file(const char* dir, const char* name, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) {
    fprintf(stderr, "cannot open %s\n", path);
    exit(2);
  }
  void* host = malloc(bytes);
  if (!host || fread(host, 1, bytes, f) != bytes) {
    fprintf(stderr, "short read: %s\n", path);
    exit(2);
  }
  fclose(f);
  return host;
}

static void write_file(const char* dir, const char* name, const void* host, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(host, 1, bytes, f) != bytes) {
    fprintf(stderr, "cannot write %s\n", path);
    exit(2);
  }
  fclose(f);
}

static void cuda_ok(cudaError_t e, const char* what) {
  if (e != cudaSuccess) {
    fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
    exit(3);
  }
}

static void vmla_ok(vmla_status s, const char* what) {
  if (s != VMLA_OK) {
    fprintf(stderr, "%s: %s (%s)\n", what, vmla_status_string(s), vmla_last_error());
    exit(4);
  }
}

/* Host file -> new device buffer. */
static uint16_t* upload(const char* dir, const char* name, size_t elems) {
  void* host = read_file(dir, name, elems * 2);
  void* dev = NULL;
  cuda_ok(cudaMalloc(&dev, elems * 2), "cudaMalloc");
  cuda_ok(cudaMemcpy(dev, host, elems * 2, cudaMemcpyHostToDevice), "cudaMemcpy H2D");
  free(host);
  return (uint16_t*)dev;
}

static void download(const char* dir, const char* name, const uint16_t* dev, size_t elems) {
  void* host = malloc(elems * 2);
  cuda_ok(cudaMemcpy(host, dev, elems * 2, cudaMemcpyDeviceToHost), "cudaMemcpy D2H");
  write_file(dir, name, host, elems * 2);
  free(host);
}

int main(int argc, char** argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: %s <dir>\n", argv[0]);
    return 1;
  }
  const char* dir = argv[1];
  char path[4096];
  snprintf(path, sizeof path, "%s/meta.txt", dir);
  FILE* f = fopen(path, "r");
  int batch, n_q, heads, d_model, grid_h, grid_w;
  long long n_kv, chunk_t0;
  float scale;
  if (!f || fscanf(f, "%d %d %lld %d %d %lld %d %d %f", &batch, &n_q, &n_kv, &heads, &d_model, &chunk_t0,
                   &grid_h, &grid_w, &scale) != 9) {
    fprintf(stderr, "bad meta.txt\n");
    return 2;
  }
  fclose(f);
  const size_t D = (size_t)d_model, H = (size_t)heads, B = (size_t)batch;
  const long long per_frame = (long long)grid_h * grid_w;
  const int frames = (int)(n_kv / per_frame);

  uint16_t* x = upload(dir, "x.bin", B * n_kv * D);
  uint16_t* w_dkv = upload(dir, "w_dkv.bin", 192 * D);
  uint16_t* w_kr = upload(dir, "w_kr.bin", 32 * D);
  uint16_t* q = upload(dir, "q.bin", B * n_q * H * 128);
  uint16_t* q_rope = upload(dir, "q_rope.bin", B * n_q * H * 32);
  uint16_t* w_uk = upload(dir, "w_uk.bin", H * 128 * 192);
  uint16_t* w_uv = upload(dir, "w_uv.bin", H * 128 * 192);
  uint16_t* k = upload(dir, "k.bin", B * n_kv * H * 128);
  uint16_t* v = upload(dir, "v.bin", B * n_kv * H * 128);
  uint16_t *cache = NULL, *out = NULL, *out_dense = NULL, *xc = NULL;
  cuda_ok(cudaMalloc((void**)&cache, B * n_kv * 224 * 2), "cudaMalloc cache");
  cuda_ok(cudaMalloc((void**)&out, B * n_q * H * 128 * 2), "cudaMalloc out");
  cuda_ok(cudaMalloc((void**)&out_dense, B * n_q * H * 128 * 2), "cudaMalloc out_dense");
  cuda_ok(cudaMalloc((void**)&xc, B * 3 * per_frame * D * 2), "cudaMalloc chunk");

  cudaStream_t stream;
  cuda_ok(cudaStreamCreate(&stream), "cudaStreamCreate");
  /* The window, 3 frames per call; a chunk's x is gathered into its own
   * [B, tokens, D] buffer, as a caller holding the chunk's hidden states would. */
  for (int f0 = 0; f0 < frames; f0 += 3) {
    const int nf = frames - f0 < 3 ? frames - f0 : 3;
    const size_t tok = (size_t)nf * per_frame;
    cuda_ok(cudaMemcpy2DAsync(xc, tok * D * 2, x + (size_t)f0 * per_frame * D, (size_t)n_kv * D * 2, tok * D * 2,
                              B, cudaMemcpyDeviceToDevice, stream),
            "gather chunk");
    vmla_ok(vmla_cache_append(xc, w_dkv, w_kr, batch, (int32_t)tok, d_model, cache, n_kv, (int64_t)f0 * per_frame,
                              f0, grid_h, grid_w, stream),
            "vmla_cache_append");
  }
  vmla_ok(vmla_chunk_attention(q, q_rope, w_uk, w_uv, cache, batch, n_q, heads, n_kv, n_kv, chunk_t0, grid_h, grid_w,
                               scale, out, stream),
          "vmla_chunk_attention");
  vmla_ok(vmla_dense_attention(q, k, v, batch, n_q, n_kv, heads, 128, scale, out_dense, stream),
          "vmla_dense_attention");
  vmla_ok(vmla_get_device_status(stream), "vmla_get_device_status");

  download(dir, "cache.bin", cache, B * n_kv * 224);
  download(dir, "out.bin", out, B * n_q * H * 128);
  download(dir, "out_dense.bin", out_dense, B * n_q * H * 128);
  printf("ok\n");
  return 0;
}
