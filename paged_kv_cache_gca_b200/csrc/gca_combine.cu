// Split-KV combine: merges the partial (O, row max, row sum) records that the attention
// kernel leaves for every (head, query tile) whose key range was cut between CTAs
// (LingBot-Map GCT page, "Attention Blocks: FlashInfer vs. SDPA": the frame's queries attend
// over the whole cache; a split attention is recombined with log-sum-exp weights).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "gca_internal.h"

namespace gca {
namespace {

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Merges the partial records of every split (head, query tile): weights 2^(m_s - M),
// M = max_s m_s. A block covers 32 query rows of one (head, query tile) with 8 threads per row,
// 8 output columns (two 16-byte loads per piece) each, so many loads are in flight per SM.
constexpr int kRowsPerBlock = 32;
constexpr int kThreadsPerRow = 8;
constexpr int kCombineThreads = kRowsPerBlock * kThreadsPerRow;
constexpr int kBlocksPerTile = kTileQ / kRowsPerBlock;
constexpr int kGroup = 4;  // pieces whose loads are issued together

// The merge of one query row (this thread's 8 columns).
__device__ __forceinline__ void merge_row(const AttnParams& p, int u2, int qq, int h, int qi,
                                          int r, int col, int64_t c0, int64_t c1,
                                          unsigned int* wide) {
  const int np = (int)(c1 - c0 + 1);
  if (np <= kGroup) {
    // the common case: every piece's (m, l) and O values in one round of loads, then the same
    // arithmetic as below (maxima first, pieces summed in CTA order)
    float2 ml[kGroup];
    float4 v[kGroup][2];
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      if (k < np) {
        const int64_t slot = part_slot(c0 + k, u2, qq);
        ml[k] = __ldcg(&p.part_ml[slot * kTileQ + r]);
        const float4* src =
            reinterpret_cast<const float4*>(p.part_o + (slot * kTileQ + r) * kHeadDim + col);
        v[k][0] = __ldcg(src);
        v[k][1] = __ldcg(src + 1);
      }
    }
    float M = -INFINITY, m_lo = INFINITY;
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      if (k < np) {
        M = fmaxf(M, ml[k].x);
        m_lo = fminf(m_lo, ml[k].x);
      }
    }
    if (col == 0 && M - m_lo > 8.0f) atomicAdd_block(wide, 1u);
    float acc[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) acc[a] = 0.f;
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      if (k >= np) break;
      const float w = ex2(ml[k].x - M);
      L += w * ml[k].y;
      acc[0] += w * v[k][0].x;
      acc[1] += w * v[k][0].y;
      acc[2] += w * v[k][0].z;
      acc[3] += w * v[k][0].w;
      acc[4] += w * v[k][1].x;
      acc[5] += w * v[k][1].y;
      acc[6] += w * v[k][1].z;
      acc[7] += w * v[k][1].w;
    }
    const float inv = 1.f / L;
    uint4 o;
    o.x = pack_bf2(acc[0] * inv, acc[1] * inv);
    o.y = pack_bf2(acc[2] * inv, acc[3] * inv);
    o.z = pack_bf2(acc[4] * inv, acc[5] * inv);
    o.w = pack_bf2(acc[6] * inv, acc[7] * inv);
    p.out[((int64_t)qi * p.H + h) * 8 + col / 8] = o;
    return;
  }
  // More pieces: read in groups so that several loads are in flight per thread; they are summed
  // in CTA order, as one at a time would.
  float M = -INFINITY, m_lo = INFINITY;
  for (int g = 0; g < np; g += kGroup) {
    float mx[kGroup];
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      mx[k] = g + k < np ? __ldcg(&p.part_ml[part_slot(c0 + g + k, u2, qq) * kTileQ + r]).x
                         : -INFINITY;
    }
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      M = fmaxf(M, mx[k]);
      if (g + k < np) m_lo = fminf(m_lo, mx[k]);
    }
  }
  if (col == 0 && M - m_lo > 8.0f) atomicAdd_block(wide, 1u);
  float acc[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) acc[a] = 0.f;
  float L = 0.f;
  for (int g = 0; g < np; g += kGroup) {
    float2 ml[kGroup];
    float4 v[kGroup][2];
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      const int64_t slot = part_slot(c0 + g + (g + k < np ? k : 0), u2, qq);
      ml[k] = __ldcg(&p.part_ml[slot * kTileQ + r]);
      const float4* src =
          reinterpret_cast<const float4*>(p.part_o + (slot * kTileQ + r) * kHeadDim + col);
      v[k][0] = __ldcg(src);
      v[k][1] = __ldcg(src + 1);
    }
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      if (g + k >= np) break;
      const float w = ex2(ml[k].x - M);
      L += w * ml[k].y;
      acc[0] += w * v[k][0].x;
      acc[1] += w * v[k][0].y;
      acc[2] += w * v[k][0].z;
      acc[3] += w * v[k][0].w;
      acc[4] += w * v[k][1].x;
      acc[5] += w * v[k][1].y;
      acc[6] += w * v[k][1].z;
      acc[7] += w * v[k][1].w;
    }
  }
  const float inv = 1.f / L;
  uint4 o;
  o.x = pack_bf2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf2(acc[6] * inv, acc[7] * inv);
  p.out[((int64_t)qi * p.H + h) * 8 + col / 8] = o;
}


__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const AttnParams p) {
  // Which pieces hold this block's rows depends on the launch parameters alone: worked out
  // before the wait, while the attention launch finishes.
  const int u = blockIdx.x / kBlocksPerTile;  // (head, query tile)
  const int r = (blockIdx.x % kBlocksPerTile) * kRowsPerBlock + threadIdx.x / kThreadsPerRow;
  const int col = (threadIdx.x % kThreadsPerRow) * 8;
  const int h = u / p.n_qt;
  const int qt = u % p.n_qt;
  const int u2 = h * p.n_pairs + qt / kQPerCta;
  const int qq = qt % kQPerCta;
  const int64_t first = (int64_t)u2 * p.n_tiles;
  const int64_t c0 = cta_of_step(first, p);
  const int64_t c1 = cta_of_step(first + p.n_tiles - 1, p);
  if (c0 == c1) return;  // not split: the attention kernel wrote these rows
  pdl_wait();             // the attention launch's partial records
  const int qi = qt * kTileQ + r;
  __shared__ unsigned int wide;  // rows of this block merged over maxima > 2^8 apart
  __shared__ unsigned int dead;  // the cache's sticky error word (read once per block)
  if (threadIdx.x == 0) {
    wide = 0u;
    dead = *reinterpret_cast<volatile uint32_t*>(p.err);
  }
  __syncthreads();
  if (dead != 0u) return;  // sticky error: no-op
  if (qi < p.T) merge_row(p, u2, qq, h, qi, r, col, c0, c1, &wide);
  __syncthreads();
  if (threadIdx.x == 0 && wide != 0u) atomicAdd(&p.counters[2], (unsigned long long)wide);
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_combine(const AttnParams& p, cudaStream_t s) {
  return launch_dependent(combine_kernel, dim3(p.units * kBlocksPerTile), dim3(kCombineThreads),
                          0, s, p);
}

}  // namespace gca
