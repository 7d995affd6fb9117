// Per-item code of the append step, shared by the append kernels of gca_append.cu: the per-frame
// kernel (four items per thread, loads hoisted) and the batched kernel (one item per thread) write
// bit-identical pages.
//
// One frame's append ("How the Geometric Context Transformer Enables Streaming 3D Reconstruction
// in LingBot-Map", FlashInferBlock: append_frame, then evict_frames) splits into items:
//   token items: one 16-byte chunk c (8 dims) of token i (a slot of the frame's pages), head h:
//     a1  the page of slot i comes from the FIFO free list (ring position free_head + i / 16);
//         slot 0 of a page records it in the frame's page-table row; slot_map[i] = page*16 +
//         i%16;
//     a2  q and k get 3D (t, y, x) RoPE ("3D Rotary Positional Embeddings"); k_rot and v go to
//         the slot with 16-byte stores, q_rot to the caller's buffer (skipped when there is
//         none); padding slots of the frame's last page are zeroed;
//   aux items:
//     a3  copies of the evicted frame's kept tokens to the trajectory tail ("How GCT's
//         Anchor-Pose-Trajectory Pools Make Monocular 3D Tractable": evicted frames keep only
//         compact context tokens), zero fill of a fresh trajectory page, pushes of the evicted
//         frame's pages to the free-list tail, records of the trajectory pages popped.
// The host mirrors every count, so the ring positions are parameters and no item waits on
// another: the pops read positions [head, head+ppf+n_traj) while the pushes write
// [tail, tail+ppf), and these never overlap because a frame is only evicted when at least
// (A+W)*ppf pages are in use.
#pragma once

#include <cuda_bf16.h>

#include "gca_internal.h"

namespace gca {
namespace append_item {

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }
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

// (cos, sin) of pair j (0..31) of token i at RoPE time position rope_frame.
__device__ __forceinline__ float2 rope_cs(const float2* rope_t, const float2* rope_tok, int nt,
                                          int nyx, int64_t rope_frame, int i, int j) {
  return j < nt ? rope_t[rope_frame * nt + j] : rope_tok[(int64_t)i * nyx + (j - nt)];
}

__device__ __forceinline__ int wrap(int pos, int n) { return pos >= n ? pos - n : pos; }

// Token item (i, h, c). The 8 chunks of one (i, h) sit in 8 consecutive lanes of a warp (lanes
// 8g .. 8g+7) and call this together (they share i, so they take the same branches). kWithQ:
// also rotate q into p.q_rot.
template <bool kWithQ>
__device__ __forceinline__ void token_chunk(const AppendParams& p, int i, int h, int c) {
  const int H = p.H;
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
  uint4 qv;
  if (kWithQ) qv = p.q[src];
  const uint4 kv = p.k[src];
  const uint4 vv = p.v[src];
  float2 cs[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    cs[w] = rope_cs(p.rope_t, p.rope_tok, p.nt, p.nyx, p.rope_frame, i, 4 * c + w);
  }
  uint4 qr, kr;
  if (kWithQ) {
    qr.x = rotate_word(qv.x, cs[0]);
    qr.y = rotate_word(qv.y, cs[1]);
    qr.z = rotate_word(qv.z, cs[2]);
    qr.w = rotate_word(qv.w, cs[3]);
  }
  kr.x = rotate_word(kv.x, cs[0]);
  kr.y = rotate_word(kv.y, cs[1]);
  kr.z = rotate_word(kv.z, cs[2]);
  kr.w = rotate_word(kv.w, cs[3]);
  if (h == 0 && c == 0) {
    p.slot_map[i] = page * kPageSize + slot;
    if (slot == 0) p.frame_pages[p.t * p.ppf + i / kPageSize] = page;
  }
  if (kWithQ) p.q_rot[src] = qr;
  p.k_pool[dst] = kr;
  p.v_pool[dst] = vv;
  // The stored key's squared norm raises the head's running maximum: the attention bounds
  // every score of a row by |q| * max|k| and skips its row max while that bound is below the
  // running max + 2^8. Computed after the stores, when the q and v registers are free.
  float ss = 0.f;
  const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float a = bf_lo(kw[w]), b = bf_hi(kw[w]);
    ss = fmaf(a, a, fmaf(b, b, ss));
  }
  unsigned lane;
  asm("mov.u32 %0, %%laneid;" : "=r"(lane));
  const unsigned group = 0xffu << (lane & 24u);
  ss += __shfl_xor_sync(group, ss, 1);
  ss += __shfl_xor_sync(group, ss, 2);
  ss += __shfl_xor_sync(group, ss, 4);
  if (c == 0 && ss > __uint_as_float(p.kmax[h])) atomicMax(&p.kmax[h], __float_as_uint(ss));
}

// Token items base + lane + 32 u, u = 0..3 (base a multiple of 8, all four below the token item
// count): the same writes as four token_chunk<kWithQ> calls, with the loads of the four items
// issued before any of their stores so that they are in flight together.
template <bool kWithQ>
__device__ __forceinline__ void token_chunks4(const AppendParams& p, int64_t base, int lane) {
  const int H = p.H;
  const int c = lane & 7;
  int i[4], h[4], page[4];
  uint4 qv[4], kv[4], vv[4];
  float2 cs[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t th = (base + 32 * u + lane) >> 3;
    h[u] = (int)(th % H);
    i[u] = (int)(th / H);
    page[u] = p.free_ring[wrap(p.head_pos + i[u] / kPageSize, p.num_pages)];
    if (i[u] < p.T) {
      const int64_t src = ((int64_t)i[u] * H + h[u]) * 8 + c;
      if (kWithQ) qv[u] = p.q[src];
      kv[u] = p.k[src];
      vv[u] = p.v[src];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        cs[u][w] = rope_cs(p.rope_t, p.rope_tok, p.nt, p.nyx, p.rope_frame, i[u], 4 * c + w);
      }
    }
  }
  unsigned lane_id;
  asm("mov.u32 %0, %%laneid;" : "=r"(lane_id));
  const unsigned group = 0xffu << (lane_id & 24u);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (page[u] < 0 || page[u] >= p.num_pages) {
      set_err(p.err, GCA_DEVERR_PAGE_RANGE);
      continue;
    }
    const int slot = i[u] % kPageSize;
    const int64_t dst = (((int64_t)page[u] * H + h[u]) * kPageSize + slot) * 8 + c;
    if (i[u] >= p.T) {  // padding slot of the frame's last page
      p.k_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
      p.v_pool[dst] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    if (kWithQ) {
      uint4 qr;
      qr.x = rotate_word(qv[u].x, cs[u][0]);
      qr.y = rotate_word(qv[u].y, cs[u][1]);
      qr.z = rotate_word(qv[u].z, cs[u][2]);
      qr.w = rotate_word(qv[u].w, cs[u][3]);
      p.q_rot[((int64_t)i[u] * H + h[u]) * 8 + c] = qr;
    }
    uint4 kr;
    kr.x = rotate_word(kv[u].x, cs[u][0]);
    kr.y = rotate_word(kv[u].y, cs[u][1]);
    kr.z = rotate_word(kv[u].z, cs[u][2]);
    kr.w = rotate_word(kv[u].w, cs[u][3]);
    if (h[u] == 0 && c == 0) {
      p.slot_map[i[u]] = page[u] * kPageSize + slot;
      if (slot == 0) p.frame_pages[p.t * p.ppf + i[u] / kPageSize] = page[u];
    }
    p.k_pool[dst] = kr;
    p.v_pool[dst] = vv[u];
    float ss = 0.f;
    const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float a = bf_lo(kw[w]), b = bf_hi(kw[w]);
      ss = fmaf(a, a, fmaf(b, b, ss));
    }
    ss += __shfl_xor_sync(group, ss, 1);
    ss += __shfl_xor_sync(group, ss, 2);
    ss += __shfl_xor_sync(group, ss, 4);
    if (c == 0 && ss > __uint_as_float(p.kmax[h[u]])) {
      atomicMax(&p.kmax[h[u]], __float_as_uint(ss));
    }
  }
}

// Aux item idx (0 <= idx < p.n_aux_items).
__device__ __forceinline__ void aux(const AppendParams& p, int64_t idx) {
  const int H = p.H;
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

}  // namespace append_item
}  // namespace gca
