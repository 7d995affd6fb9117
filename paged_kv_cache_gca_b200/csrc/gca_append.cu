// Append-side kernels of the GCA paged KV cache (sm_100a).
//
// append_kernel does one frame's whole append step in a single launch (the per-item code and
// its description are in gca_append_item.cuh), following the order of the pages' streaming
// block ("How the Geometric Context Transformer Enables Streaming 3D
// Reconstruction in LingBot-Map", FlashInferBlock: append_frame, then evict_frames):
//   a1  the frame's pages are popped from the FIFO free list (ring positions free_head ..
//       free_head+ppf-1) and written to its page-table row; slot_map[i] = page*16 + i%16;
//   a2  q and k get 3D (t, y, x) RoPE ("3D Rotary Positional Embeddings"); k_rot and v go to
//       their slots with 16-byte stores, q_rot to the caller's buffer; the unused slots of the
//       frame's last page are zeroed;
//   a3  the frame leaving the window hands its kept tokens to the trajectory tail ("How GCT's
//       Anchor-Pose-Trajectory Pools Make Monocular 3D Tractable": evicted frames keep only
//       compact context tokens), new trajectory pages come from ring positions right after the
//       frame's, and the evicted frame's pages go to the ring tail.
// The host mirrors every count, so the ring positions are kernel arguments and no block waits
// on another: the pops read positions [head, head+ppf+n_traj) while the pushes write
// [tail, tail+ppf), and these never overlap because a frame is only evicted when at least
// (A+W)*ppf pages are in use.
#include <cuda_bf16.h>

#include "gca_append_item.cuh"

namespace gca {

namespace {

constexpr int kThreads = 256;

using append_item::set_err;

// ------------------------------------------------------------------------------- init

__global__ void init_kernel(const InitParams p) {
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // free list and its saved copy; count occurrences for the permutation check
  for (int64_t i = tid; i < p.num_pages; i += stride) {
    int32_t v = p.user_free ? p.user_free[i] : (int32_t)i;
    p.free_ring[i] = v;
    p.init_free[i] = v;
    if (v >= 0 && v < p.num_pages) {
      atomicAdd(&p.seen[v], 1);
    } else {
      set_err(p.err, GCA_DEVERR_FREE_LIST);
    }
  }
  for (int64_t i = tid; i < p.keep; i += stride) p.kept[i] = p.kept_host[i];
  // RoPE tables in fp64, stored as fp32 (cos, sin): pair j of a band of width d turns by
  // pos * base^(-2j/d). Time band per frame; the two spatial bands per token (camera/register
  // tokens at (y, x) = (0, 0), the patch at row r, column c at (r+1, c+1)).
  const int64_t n_t = (int64_t)p.max_frames * p.nt;
  const int nyx = p.ny + p.nx;
  const int64_t n_s = (int64_t)p.T * nyx;
  for (int64_t i = tid; i < n_t + n_s; i += stride) {
    int64_t pos, j;
    int d;
    float2* dst;
    if (i < n_t) {
      pos = i / p.nt;
      j = i % p.nt;
      d = 2 * p.nt;
      dst = p.rope_t + i;
    } else {
      const int64_t r = i - n_t;
      const int64_t tok = r / nyx;
      const int64_t pr = r % nyx;  // pair index within the spatial bands
      int64_t y = 0, x = 0;
      if (tok >= p.num_special) {
        y = (tok - p.num_special) / p.grid_w + 1;
        x = (tok - p.num_special) % p.grid_w + 1;
      }
      if (pr < p.ny) {
        pos = y;
        j = pr;
        d = 2 * p.ny;
      } else {
        pos = x;
        j = pr - p.ny;
        d = 2 * p.nx;
      }
      dst = p.rope_tok + r;
    }
    const double inv_freq = pow(p.base, -2.0 * (double)j / (double)d);
    const double ang = (double)pos * inv_freq;
    double sn, cs;
    sincos(ang, &sn, &cs);
    *dst = make_float2((float)cs, (float)sn);
  }
}

__global__ void check_perm_kernel(const int32_t* seen, uint32_t* err, int32_t n) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < n && seen[i] != 1) set_err(err, GCA_DEVERR_FREE_LIST);
}

__global__ void reset_kernel(int32_t* free_ring, const int32_t* init_free, uint32_t* err,
                             int32_t n) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < n) free_ring[i] = init_free[i];
  if (i == 0) *err = 0u;
}

// ------------------------------------------------------------------------------- append

// Block bx of one cache's append. Token part: block (8 chunks, H heads, tok_per_block tokens);
// one thread = one 16-byte chunk (8 dims) of one (token, head). Auxiliary part (blocks after
// n_tok_blocks): eviction copies, zero fill of a fresh trajectory page, free-list pushes,
// trajectory page records.
__device__ __forceinline__ void append_block(const AppendParams& p, const int bx) {
  const int H = p.H;
  // The append does not test the sticky error word (that costs ~10% of its bandwidth through
  // register pressure): every page id is range-checked before any write, so it stays in
  // bounds, and the attention and combine kernels, which do test the word, write no output.
  if (bx < p.n_tok_blocks) {
    const int i = bx * p.tok_per_block + threadIdx.z;
    if (i >= p.ppf * kPageSize) return;
    // the 8 chunks of one (token, head) are 8 consecutive lanes (threads are linearised x first)
    append_item::token_chunk<true>(p, i, threadIdx.y, threadIdx.x);
    return;
  }
  const int block_threads = 8 * H * p.tok_per_block;
  const int lin = threadIdx.x + 8 * (threadIdx.y + H * threadIdx.z);
  const int64_t idx = (int64_t)(bx - p.n_tok_blocks) * block_threads + lin;
  if (idx < p.n_aux_items) append_item::aux(p, idx);
}

// At most 512 threads (8 chunks x 64 heads) and 32 registers: 8 blocks of 256 threads per SM
// (the append is a latency-bound copy and wants every warp it can get: 6 blocks measured 5%
// slower).
#define GCA_APPEND_BOUNDS __launch_bounds__(512, 4)

// One frame's append: warp w of the grid takes token items [128 w, 128 w + 128), four per lane
// with their loads in flight together (a single 12 MB frame is one short wave, so memory-level
// parallelism per thread, not occupancy, bounds it); the warps after the token items take the
// eviction items, one per lane.
constexpr int kAppendWarpsPerBlock = 8;
constexpr int kItemsPerWarp = 128;

__global__ void __launch_bounds__(32 * kAppendWarpsPerBlock)
    append_kernel(const AppendParams p) {
  pdl_wait();  // inputs, pages and the free ring may come from earlier work in the stream
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * kAppendWarpsPerBlock + (threadIdx.x >> 5);
  const int64_t n_tok = (int64_t)p.ppf * kPageSize * p.H * 8;
  const int64_t tok_warps = n_tok / kItemsPerWarp;
  if (warp < tok_warps) {
    append_item::token_chunks4<true>(p, warp * kItemsPerWarp, lane);
  } else {
    const int64_t idx = (warp - tok_warps) * 32 + lane;
    if (idx < p.n_aux_items) append_item::aux(p, idx);
  }
  pdl_launch_dependents();
}

__global__ void GCA_APPEND_BOUNDS append_batch_kernel(const __grid_constant__ AppendBatch b) {
  pdl_wait();
  const AppendParams& p = b.p[blockIdx.y];
  if ((int)blockIdx.x < p.n_blocks) append_block(p, (int)blockIdx.x);
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_init(const InitParams& p, cudaStream_t s) {
  int64_t work = p.num_pages;
  const int64_t rope = (int64_t)p.max_frames * p.nt + (int64_t)p.T * (p.ny + p.nx);
  if (rope > work) work = rope;
  int64_t blocks = (work + kThreads - 1) / kThreads;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  init_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_check_perm(int32_t* seen, uint32_t* err, int32_t n, cudaStream_t s) {
  check_perm_kernel<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(seen, err, n);
  return cudaGetLastError();
}

cudaError_t launch_reset(int32_t* free_ring, const int32_t* init_free, uint32_t* err,
                         int32_t n, cudaStream_t s) {
  reset_kernel<<<(n + kThreads - 1) / kThreads, kThreads, 0, s>>>(free_ring, init_free, err, n);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  // token items: ppf * 16 slots x H heads x 8 chunks, a multiple of 128 since 16 * 8 = 128
  const int64_t n_tok = (int64_t)p.ppf * kPageSize * p.H * 8;
  const int64_t warps = n_tok / kItemsPerWarp + (p.n_aux_items + 31) / 32;
  const int64_t blocks = (warps + kAppendWarpsPerBlock - 1) / kAppendWarpsPerBlock;
  return launch_dependent(append_kernel, dim3((unsigned)blocks),
                          dim3(32 * kAppendWarpsPerBlock), 0, s, p);
}

cudaError_t launch_append_batch(const AppendBatch& b, cudaStream_t s) {
  const dim3 block(8, b.p[0].H, b.p[0].tok_per_block);
  return launch_dependent(append_batch_kernel, dim3((unsigned)b.max_blocks, (unsigned)b.n), block,
                          0, s, b);
}

}  // namespace gca
