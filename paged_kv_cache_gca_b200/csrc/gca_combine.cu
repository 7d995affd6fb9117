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
// M = max_s m_s. Two threads per query row, 32 output columns each.
constexpr int kCombineThreads = 2 * kTileQ;
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const AttnParams p) {
  pdl_signal_early();
  pdl_wait();  // the attention launch's partial records
  if (*reinterpret_cast<volatile uint32_t*>(p.err) != 0u) return;  // sticky error: no-op
  const int u = blockIdx.x;  // (head, query tile)
  const int r = threadIdx.x >> 1;
  const int half = threadIdx.x & 1;
  const int h = u / p.n_qt;
  const int qt = u % p.n_qt;
  const int u2 = h * p.n_pairs + qt / kQPerCta;
  const int qq = qt % kQPerCta;
  const int64_t first = (int64_t)u2 * p.n_tiles;
  const int64_t c0 = cta_of_step(first, p.total, p.grid);
  const int64_t c1 = cta_of_step(first + p.n_tiles - 1, p.total, p.grid);
  if (c0 == c1) return;
  const int qi = qt * kTileQ + r;
  if (qi >= p.T) return;
  // Pieces are read in groups so that several loads are in flight per thread; they are summed
  // in CTA order, as one at a time would.
  const int np = (int)(c1 - c0 + 1);
  float M = -INFINITY;
  for (int g = 0; g < np; g += 4) {
    float mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mx[k] = g + k < np ? __ldcg(&p.part_ml[part_slot(c0 + g + k, u2, qq) * kTileQ + r]).x
                         : -INFINITY;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) M = fmaxf(M, mx[k]);
  }
  float acc[32];
#pragma unroll
  for (int a = 0; a < 32; ++a) acc[a] = 0.f;
  float L = 0.f;
  for (int g = 0; g < np; g += 2) {
    float2 ml[2];
    float4 v[2][8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t slot = part_slot(c0 + g + (g + k < np ? k : 0), u2, qq);
      ml[k] = __ldcg(&p.part_ml[slot * kTileQ + r]);
      const float4* src =
          reinterpret_cast<const float4*>(p.part_o + (slot * kTileQ + r) * kHeadDim + 32 * half);
#pragma unroll
      for (int a = 0; a < 8; ++a) v[k][a] = __ldcg(src + a);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (g + k >= np) break;
      const float w = ex2(ml[k].x - M);
      L += w * ml[k].y;
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        acc[4 * a] += w * v[k][a].x;
        acc[4 * a + 1] += w * v[k][a].y;
        acc[4 * a + 2] += w * v[k][a].z;
        acc[4 * a + 3] += w * v[k][a].w;
      }
    }
  }
  const float inv = 1.f / L;
  uint4* dst = p.out + ((int64_t)qi * p.H + h) * 8 + 4 * half;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 w;
    w.x = pack_bf2(acc[8 * c + 0] * inv, acc[8 * c + 1] * inv);
    w.y = pack_bf2(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
    w.z = pack_bf2(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
    w.w = pack_bf2(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
    dst[c] = w;
  }
  pdl_signal_late();
}

}  // namespace

cudaError_t launch_combine(const AttnParams& p, cudaStream_t s) {
  return launch_dependent(combine_kernel, dim3(p.units), dim3(kCombineThreads), 0, s, p);
}

}  // namespace gca
