// Append-side kernels of the GCA paged KV cache (sm_100a).
//
// gca_append_kernel does one frame's whole append step in a single launch, following the order
// of the pages' streaming block ("How the Geometric Context Transformer Enables Streaming 3D
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

#include "gca_internal.h"

namespace gca {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

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

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Rotates the pair held in one 32-bit word (element 2j in the low half, 2j+1 in the high half).
__device__ __forceinline__ uint32_t rotate_word(uint32_t w, float2 cs) {
  const float a = bf_lo(w), b = bf_hi(w);
  const float ra = fmaf(a, cs.x, -b * cs.y);
  const float rb = fmaf(a, cs.y, b * cs.x);
  return pack_bf2(ra, rb);
}

__device__ __forceinline__ int wrap(int pos, int n) { return pos >= n ? pos - n : pos; }


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
    // ---- a1 + a2
    const int c = threadIdx.x;
    const int h = threadIdx.y;
    const int i = bx * p.tok_per_block + threadIdx.z;
    if (i >= p.ppf * kPageSize) return;
    const int page = p.free_ring[wrap(p.head_pos + i / kPageSize, p.num_pages)];
    if (page < 0 || page >= p.num_pages) {
      set_err(p.err, GCA_DEVERR_PAGE_RANGE);
      return;
    }
    const int slot = i % kPageSize;
    const int64_t dst = (((int64_t)page * H + h) * kPageSize + slot) * 8 + c;
    if (i >= p.T) {  // padding slot of the frame's last page
      p.k_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.v_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
      return;
    }
    const int64_t src = ((int64_t)i * H + h) * 8 + c;
    const uint4 qv = p.q[src];
    const uint4 kv = p.k[src];
    const uint4 vv = p.v[src];
    float2 cs[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = 4 * c + w;  // pair index within the head
      cs[w] = j < p.nt ? p.rope_t[p.rope_frame * p.nt + j]
                     : p.rope_tok[(int64_t)i * p.nyx + (j - p.nt)];
    }
    uint4 qr, kr;
    qr.x = rotate_word(qv.x, cs[0]);
    qr.y = rotate_word(qv.y, cs[1]);
    qr.z = rotate_word(qv.z, cs[2]);
    qr.w = rotate_word(qv.w, cs[3]);
    kr.x = rotate_word(kv.x, cs[0]);
    kr.y = rotate_word(kv.y, cs[1]);
    kr.z = rotate_word(kv.z, cs[2]);
    kr.w = rotate_word(kv.w, cs[3]);
    if (h == 0 && c == 0) {
      p.slot_map[i] = page * kPageSize + slot;
      if (slot == 0) p.frame_pages[p.t * p.ppf + i / kPageSize] = page;
    }
    p.q_rot[src] = qr;
    p.k_pool[dst] = kr;
    p.v_pool[dst] = vv;
    // The stored key's squared norm raises the head's running maximum: the attention bounds
    // every score of a row by |q| * max|k| and skips its row max while that bound is below
    // the running max + 2^8. Computed after the stores, when the q and v registers are free.
    {
      float ss = 0.f;
      const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float a = bf_lo(kw[w]), b = bf_hi(kw[w]);
        ss = fmaf(a, a, fmaf(b, b, ss));
      }
      // the 8 chunks of one (token, head) are 8 consecutive lanes
      const unsigned lane = (threadIdx.x + 8u * (threadIdx.y + (unsigned)H * threadIdx.z)) & 31u;
      const unsigned group = 0xffu << (lane & 24u);
      ss += __shfl_xor_sync(group, ss, 1);
      ss += __shfl_xor_sync(group, ss, 2);
      ss += __shfl_xor_sync(group, ss, 4);
      if (c == 0 && ss > __uint_as_float(p.kmax[h])) atomicMax(&p.kmax[h], __float_as_uint(ss));
    }
    return;
  }

  const int block_threads = 8 * H * p.tok_per_block;
  const int lin = threadIdx.x + 8 * (threadIdx.y + H * threadIdx.z);
  const int64_t idx = (int64_t)(bx - p.n_tok_blocks) * block_threads + lin;
  if (idx >= p.n_aux_items) return;
  const int64_t e_ev = p.n_evict_items;
  const int64_t e_zero = e_ev + p.n_zero_items;
  const int64_t e_push = e_zero + p.n_push_items;
  const int first_new = wrap(p.head_pos + p.ppf, p.num_pages);  // first trajectory pop

  if (idx < e_ev) {
    // ---- a3: copy kept token j of the evicted frame to trajectory position traj_len + j
    const int c = (int)(idx & 7);
    const int64_t th = idx >> 3;
    const int h = (int)(th % H);
    const int j = (int)(th / H);
    const int tok = p.kept[j];
    const int src_page = p.frame_pages[(int64_t)p.evict_frame * p.ppf + tok / kPageSize];
    const int64_t pos = p.traj_len + j;
    const int64_t tp = pos / kPageSize;
    const int dst_page =
        tp < p.traj_pages_before
            ? p.traj_pages[tp]
            : p.free_ring[wrap(first_new + (int)(tp - p.traj_pages_before), p.num_pages)];
    if (src_page < 0 || src_page >= p.num_pages || dst_page < 0 || dst_page >= p.num_pages) {
      set_err(p.err, GCA_DEVERR_PAGE_RANGE);
      return;
    }
    const int64_t src = (((int64_t)src_page * H + h) * kPageSize + tok % kPageSize) * 8 + c;
    const int64_t dst = (((int64_t)dst_page * H + h) * kPageSize + pos % kPageSize) * 8 + c;
    p.k_pool[dst] = p.k_pool[src];
    p.v_pool[dst] = p.v_pool[src];
    return;
  }

  if (idx < e_zero) {
    // ---- zero the slots of the last new trajectory page that this step leaves empty
    const int64_t r = idx - e_ev;
    const int c = (int)(r & 7);
    const int64_t th = r >> 3;
    const int h = (int)(th % H);
    const int z = (int)(th / H);
    const int64_t pos = p.traj_len + p.K + z;
    const int64_t tp = pos / kPageSize;
    const int page =
        p.free_ring[wrap(first_new + (int)(tp - p.traj_pages_before), p.num_pages)];
    if (page < 0 || page >= p.num_pages) {
      set_err(p.err, GCA_DEVERR_PAGE_RANGE);
      return;
    }
    const int64_t dst = (((int64_t)page * H + h) * kPageSize + pos % kPageSize) * 8 + c;
    p.k_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
    p.v_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }

  if (idx < e_push) {
    // ---- push the evicted frame's pages to the free-list tail, in row order
    const int k = (int)(idx - e_zero);
    p.free_ring[wrap(p.tail_pos + k, p.num_pages)] =
        p.frame_pages[(int64_t)p.evict_frame * p.ppf + k];
    return;
  }

  // ---- record the trajectory pages popped by this step
  const int k = (int)(idx - e_push);
  p.traj_pages[p.traj_pages_before + k] = p.free_ring[wrap(first_new + k, p.num_pages)];
}

// At most 512 threads (8 chunks x 64 heads) and 32 registers: 8 blocks of 256 threads per SM
// (the append is a latency-bound copy and wants every warp it can get: 6 blocks measured 5%
// slower).
#define GCA_APPEND_BOUNDS __launch_bounds__(512, 4)

__global__ void GCA_APPEND_BOUNDS append_kernel(const AppendParams p) {
  pdl_wait();  // inputs, pages and the free ring may come from earlier work in the stream
  append_block(p, (int)blockIdx.x);
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
  const dim3 block(8, p.H, p.tok_per_block);
  return launch_dependent(append_kernel, dim3((unsigned)p.n_blocks), block, 0, s, p);
}

cudaError_t launch_append_batch(const AppendBatch& b, cudaStream_t s) {
  const dim3 block(8, b.p[0].H, b.p[0].tok_per_block);
  return launch_dependent(append_batch_kernel, dim3((unsigned)b.max_blocks, (unsigned)b.n), block,
                          0, s, b);
}

}  // namespace gca
