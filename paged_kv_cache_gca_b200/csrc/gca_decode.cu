// Attention of a small query set (at most kDecodeMaxRows rows per head) over the keys of the
// three pools, on CUDA cores. This is the regime of the causal camera head's cache, one camera
// token per frame attending over every earlier frame's camera token ("How the Geometric Context
// Transformer Enables Streaming 3D Reconstruction in LingBot-Map", Streaming Inference API; the
// camera head keeps its own causal KV cache per trunk layer). It computes the same thing as the
// tensor-core kernel, out[i][h] = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j over the same
// logical key order, but a 128-row MMA tile would be almost all padding here.
//
// Grid (dsplit, H) in clusters of (dsplit, 1, 1): the dsplit CTAs of a head form one cluster.
// CTA (s, h) takes the logical pages [s*n/dsplit, (s+1)*n/dsplit) of head h; its 8 warps take
// every 8th page. In a warp, lane 2k+e holds key k of the page (16 slots) and dims [32e, 32e+32);
// the two lanes of a key add their halves of q.k, the warp keeps an online softmax per query row
// (row max in log2 units, row sum; lane l accumulates output dims 2l and 2l+1 from coalesced
// 128-byte V rows, loaded together with the keys). Each CTA merges its warps with log-sum-exp
// weights and stores the result into its own slot of CTA 0's shared memory (distributed shared
// memory; a cluster barrier arrived at on entry and waited for before the stores makes sure CTA
// 0 has started); after one cluster barrier CTA 0 merges the slots in rank order from its own
// shared memory and writes the output. One launch, no global scratch, and the result does not
// depend on CTA timing.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "gca_internal.h"

namespace gca {
namespace {

// Warps per CTA. 8 keeps two to three CTAs resident per SM, so a launch of 8 splits x 32 heads
// is one wave (16 warps hold an SM per CTA and took twice as long).
template <int kRows>
__host__ __device__ constexpr int decode_warps() {
  return 8;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int kRows>
__global__ void __launch_bounds__(32 * decode_warps<kRows>()) decode_kernel(const AttnParams p) {
  constexpr int kDecodeWarps = decode_warps<kRows>();
  namespace cg = cooperative_groups;
  pdl_wait();  // the append that wrote this frame's keys and the page table
  cg::cluster_group cluster = cg::this_cluster();
  const int h = blockIdx.y;
  const int split = (int)cluster.block_rank();
  const int n_split = (int)cluster.num_blocks();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int key = lane >> 1;  // slot of the page this lane's pair owns
  const int half = lane & 1;  // which 32 dims of the key and of q

  __shared__ float sm_m[kDecodeWarps][kRows];
  __shared__ float sm_l[kDecodeWarps][kRows];
  __shared__ float sm_o[kDecodeWarps][kRows][kHeadDim];
  // CTA 0's slots for every CTA's merged result (written remotely by each CTA)
  __shared__ float cl_m[kDecodeMaxSplit][kRows], cl_l[kDecodeMaxSplit][kRows];
  __shared__ float cl_o[kDecodeMaxSplit][kRows][kHeadDim];
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // Sticky error: no output until gca_reset. Every CTA still takes part in the cluster
  // barriers. The word, q and the first page ids are loaded together.
  const bool live = *reinterpret_cast<volatile uint32_t*>(p.err) == 0u;

  // this lane's 32 dims of every query row, as bf16 pairs
  uint32_t qv[kRows][16];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const uint4* src = p.q + ((int64_t)r * p.H + h) * 8 + 4 * half;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = src[c];
      qv[r][4 * c + 0] = v.x;
      qv[r][4 * c + 1] = v.y;
      qv[r][4 * c + 2] = v.z;
      qv[r][4 * c + 3] = v.w;
    }
  }

  float m_run[kRows], l_run[kRows], o0[kRows], o1[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
    o0[r] = 0.f;
    o1[r] = 0.f;
  }

  const int lp0 = (int)((int64_t)split * p.n_lp / n_split);
  const int lp1_all = (int)((int64_t)(split + 1) * p.n_lp / n_split);
  // the page id of the warp's next page is read while the current page is processed
  int next_page = 0, next_len = 0;
  if (lp0 + warp < lp1_all) resolve_page(p, lp0 + warp, 0, &next_page, &next_len);
  const int lp1 = live ? lp1_all : lp0;
  for (int lp = lp0 + warp; lp < lp1; lp += kDecodeWarps) {
    const int page = next_page, len = next_len;
    if (lp + kDecodeWarps < lp1) resolve_page(p, lp + kDecodeWarps, 0, &next_page, &next_len);
    if (page < 0 || page >= p.num_pages) {  // the same for every lane of the warp
      if (lane == 0) atomicOr(p.err, GCA_DEVERR_PAGE_RANGE);
      continue;
    }
    const int64_t row0 = ((int64_t)page * p.H + h) * kPageSize;  // slot 0 of the (page, head) block
    const bool valid = key < len;

    // this lane's keys and values of the page, loaded together
    uint4 k4[4];
    const uint4* kr = p.k_pool + (row0 + key) * 8 + 4 * half;
#pragma unroll
    for (int c = 0; c < 4; ++c) k4[c] = valid ? __ldg(kr + c) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t vv[kPageSize];
    const uint32_t* vrow = reinterpret_cast<const uint32_t*>(p.v_pool + row0 * 8) + lane;
#pragma unroll
    for (int j = 0; j < kPageSize; ++j) vv[j] = j < len ? __ldg(vrow + j * (kHeadDim / 2)) : 0u;

    // q . k over this lane's 32 dims, then over the pair
    float s[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) s[r] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t kw[4] = {k4[c].x, k4[c].y, k4[c].z, k4[c].w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          s[r] = fmaf(lo_bf16(qv[r][4 * c + w]), lo_bf16(kw[w]), s[r]);
          s[r] = fmaf(hi_bf16(qv[r][4 * c + w]), hi_bf16(kw[w]), s[r]);
        }
      }
    }
    float pk[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 1);
      const float sc = valid ? s[r] * p.scale_log2 : -INFINITY;
      float mt = sc;
#pragma unroll
      for (int off = 2; off < 32; off *= 2) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m_run[r], mt);  // finite once a page with a valid slot was seen
      const float alpha = m_new == -INFINITY ? 1.f : ex2(m_run[r] - m_new);
      pk[r] = valid ? ex2(sc - m_new) : 0.f;
      float ps = half == 0 ? pk[r] : 0.f;  // one lane per key
#pragma unroll
      for (int off = 1; off < 32; off *= 2) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l_run[r] = l_run[r] * alpha + ps;
      o0[r] *= alpha;
      o1[r] *= alpha;
      m_run[r] = m_new;
    }
    // O += P V (slots past len hold zero weight and zero values)
#pragma unroll
    for (int j = 0; j < kPageSize; ++j) {
      const float v0 = lo_bf16(vv[j]), v1 = hi_bf16(vv[j]);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const float pj = __shfl_sync(0xffffffffu, pk[r], 2 * j);
        o0[r] = fmaf(pj, v0, o0[r]);
        o1[r] = fmaf(pj, v1, o1[r]);
      }
    }
  }

  // merge the warps of the CTA
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (lane == 0) {
      sm_m[warp][r] = m_run[r];
      sm_l[warp][r] = l_run[r];
    }
    sm_o[warp][r][2 * lane] = o0[r];
    sm_o[warp][r][2 * lane + 1] = o1[r];
  }
  __syncthreads();
  const int t_row = threadIdx.x / kHeadDim;  // row and dim this thread merges
  const int t_dim = threadIdx.x % kHeadDim;
  const bool merger = threadIdx.x < kRows * kHeadDim;
  float M = -INFINITY, L = 0.f, O = 0.f;
  if (merger) {
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm_m[w][t_row]);
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float mw = sm_m[w][t_row];
      const float wt = mw == -INFINITY ? 0.f : ex2(mw - M);  // warps without keys weigh nothing
      L = fmaf(wt, sm_l[w][t_row], L);
      O = fmaf(wt, sm_o[w][t_row][t_dim], O);
    }
  }
  // every CTA of the cluster has started (its arrival on entry), so CTA 0's shared memory
  // exists: this CTA's result goes into its slot there
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (merger) {
    *cluster.map_shared_rank(&cl_o[split][t_row][t_dim], 0) = O;
    if (t_dim == 0) {
      *cluster.map_shared_rank(&cl_m[split][t_row], 0) = M;
      *cluster.map_shared_rank(&cl_l[split][t_row], 0) = L;
    }
  }
  // every CTA's result is in CTA 0's shared memory (release / acquire)
  cluster.sync();
  if (split == 0 && merger && live) {
    float Mc = -INFINITY;
    for (int c = 0; c < n_split; ++c) Mc = fmaxf(Mc, cl_m[c][t_row]);
    float Lc = 0.f, Oc = 0.f;
    for (int c = 0; c < n_split; ++c) {
      const float mc = cl_m[c][t_row];
      const float wt = mc == -INFINITY ? 0.f : ex2(mc - Mc);  // splits without keys
      Lc = fmaf(wt, cl_l[c][t_row], Lc);
      Oc = fmaf(wt, cl_o[c][t_row][t_dim], Oc);
    }
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
    out[((int64_t)t_row * p.H + h) * kHeadDim + t_dim] = __float2bfloat16_rn(Oc / Lc);
  }
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_decode(const AttnParams& p, cudaStream_t s) {
  void (*kernel)(const AttnParams) = nullptr;
  int warps = 0;
  switch (p.T) {
    case 1: kernel = decode_kernel<1>; warps = decode_warps<1>(); break;
    case 2: kernel = decode_kernel<2>; warps = decode_warps<2>(); break;
    case 3: kernel = decode_kernel<3>; warps = decode_warps<3>(); break;
    case 4: kernel = decode_kernel<4>; warps = decode_warps<4>(); break;
    default: return cudaErrorInvalidValue;
  }
  if (p.dsplit < 1 || p.dsplit > kDecodeMaxSplit) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.dsplit, p.H);
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;  // the splits of a head: one cluster
  attr[1].val.clusterDim.x = (unsigned)p.dsplit;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace gca
