/* Plain C client of the whole path through the library's C ABI, with the CUDA runtime for device
 * memory and no other framework: creates a small cache (T = 68: 8 x 8 patches + 4 special tokens,
 * 2 heads of 64, anchor 1, window 2, 4 kept tokens, permuted page order), streams 6 frames through
 * gca_append_frame + gca_attend, and writes every frame's inputs and output to a file:
 *   per frame: q, k, v, out, each bf16 [T][H][64] (uint16 bit patterns, little endian).
 * The inputs come from a 64-bit linear congruential generator (uniform in [-1, 1), rounded to
 * bf16), so tests/test_gpu_abi_c.py can feed the same values to the oracle.
 * Usage: abi_gpu <output file>. Exit status 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "gca.h"

enum { H = 2, D = 64, GRID = 8, SPECIAL = 4, T = SPECIAL + GRID * GRID, FRAMES = 6, PAGES = 24 };

static uint64_t lcg_state = 0x9E3779B97F4A7C15ull;

static uint16_t next_bf16(void) {
  lcg_state = lcg_state * 6364136223846793005ull + 1442695040888963407ull;
  const float u = (float)(lcg_state >> 40) / (float)(1u << 24) * 2.0f - 1.0f;  /* [-1, 1) */
  uint32_t bits;
  memcpy(&bits, &u, 4);
  bits += 0x7fffu + ((bits >> 16) & 1u);  /* round to nearest even */
  return (uint16_t)(bits >> 16);
}

#define CHECK_CUDA(x)                                              \
  do {                                                             \
    cudaError_t e_ = (x);                                          \
    if (e_ != cudaSuccess) {                                       \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));     \
      return 2;                                                    \
    }                                                              \
  } while (0)

#define CHECK_GCA(x)                                               \
  do {                                                             \
    gca_status s_ = (x);                                           \
    if (s_ != GCA_OK) {                                            \
      fprintf(stderr, "%s: %s\n", #x, gca_status_string(s_));      \
      return 3;                                                    \
    }                                                              \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: %s <output file>\n", argv[0]);
    return 1;
  }
  gca_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.num_heads = H;
  cfg.head_dim = D;
  cfg.page_size = 16;
  cfg.grid_h = GRID;
  cfg.grid_w = GRID;
  cfg.num_special = SPECIAL;
  cfg.anchor_frames = 1;
  cfg.window_frames = 2;
  cfg.keep_tokens = 4;
  cfg.max_frames = 8;
  cfg.num_pages = PAGES;
  cfg.rope_base = 10000.0f;
  CHECK_GCA(gca_validate_config(&cfg));

  const size_t ws_bytes = gca_workspace_bytes(&cfg);
  void* ws_alloc = NULL;  /* the workspace must start on a 1024-byte boundary */
  CHECK_CUDA(cudaMalloc(&ws_alloc, ws_bytes + 1024));
  void* ws = (void*)(((uintptr_t)ws_alloc + 1023u) & ~(uintptr_t)1023u);
  /* initial free list: pages in the order 5, 12, 19, ... (7 * i + 5 mod 24 is a permutation) */
  int32_t free_host[PAGES];
  for (int i = 0; i < PAGES; ++i) free_host[i] = (7 * i + 5) % PAGES;
  int32_t* free_dev = NULL;
  CHECK_CUDA(cudaMalloc((void**)&free_dev, sizeof(free_host)));
  CHECK_CUDA(cudaMemcpy(free_dev, free_host, sizeof(free_host), cudaMemcpyHostToDevice));

  cudaStream_t stream;
  CHECK_CUDA(cudaStreamCreate(&stream));
  gca_cache* cache = NULL;
  CHECK_GCA(gca_cache_create(&cfg, ws, ws_bytes, free_dev, stream, &cache));

  const size_t n = (size_t)T * H * D;
  const size_t bytes = n * sizeof(uint16_t);
  uint16_t* host = (uint16_t*)malloc(4 * bytes);  /* q, k, v, out */
  void *q, *k, *v, *q_rot, *out;
  CHECK_CUDA(cudaMalloc(&q, bytes));
  CHECK_CUDA(cudaMalloc(&k, bytes));
  CHECK_CUDA(cudaMalloc(&v, bytes));
  CHECK_CUDA(cudaMalloc(&q_rot, bytes));
  CHECK_CUDA(cudaMalloc(&out, bytes));
  FILE* f = fopen(argv[1], "wb");
  if (!f || !host) return 4;
  for (int t = 0; t < FRAMES; ++t) {
    for (size_t i = 0; i < 3 * n; ++i) host[i] = next_bf16();
    CHECK_CUDA(cudaMemcpyAsync(q, host, bytes, cudaMemcpyHostToDevice, stream));
    CHECK_CUDA(cudaMemcpyAsync(k, host + n, bytes, cudaMemcpyHostToDevice, stream));
    CHECK_CUDA(cudaMemcpyAsync(v, host + 2 * n, bytes, cudaMemcpyHostToDevice, stream));
    CHECK_GCA(gca_append_frame(cache, t, q, k, v, q_rot, stream));
    CHECK_GCA(gca_attend(cache, t, q_rot, out, stream));
    CHECK_CUDA(cudaMemcpyAsync(host + 3 * n, out, bytes, cudaMemcpyDeviceToHost, stream));
    CHECK_CUDA(cudaStreamSynchronize(stream));
    if (fwrite(host, 1, 4 * bytes, f) != 4 * bytes) return 5;
  }
  fclose(f);
  CHECK_GCA(gca_check(cache));  /* sticky device error word clear */
  gca_state st;
  CHECK_GCA(gca_get_state(cache, &st));
  if (st.frames_appended != FRAMES) return 6;
  CHECK_GCA(gca_cache_destroy(cache));
  cudaFree(q);
  cudaFree(k);
  cudaFree(v);
  cudaFree(q_rot);
  cudaFree(out);
  cudaFree(free_dev);
  cudaFree(ws_alloc);
  cudaStreamDestroy(stream);
  free(host);
  printf("ok %d frames\n", FRAMES);
  return 0;
}
