// Paged flash-attention forward for GCA on sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes: for every head h and query row i of the last appended frame,
//   out[i][h] = sum_j softmax_j(q_rot[i][h] . k_j[h] / sqrt(D)) v_j[h]
// over the keys of the three pools -- anchor frame(s), the window of recent frames and the
// trajectory pool ("LingBot-Map runs 10,000 frames on monocular video", section "How GCT's
// Anchor-Pose-Trajectory Pools Make Monocular 3D Tractable"; "How the Geometric Context
// Transformer Enables Streaming 3D Reconstruction in LingBot-Map", FlashInferBlock:
// compute_attention). All of a frame's queries see the same key set (frame-causal attention,
// same page, FAQ on scale frames), so the only mask is the one that hides unused page slots.
//
// Logical key order: anchor pages, window pages, trajectory pages; page lp -> physical page via
// the page table. A 96-key tile is 6 pages; each page of one head is a contiguous 2 KB block
// [16 slots][64 dims] bf16 that TMA copies into shared memory with the 128-byte swizzle.
//
// Work split: a CTA works on two 128-query tiles of one head at once (they see the same keys,
// so every K/V tile is fetched once for both); a (head, tile pair) is a work unit. The flattened
// (unit, key tile) steps are cut into `grid` contiguous ranges, one per CTA (one CTA per SM), of
// equal cost: a CTA that moves on to another unit gets fewer key tiles (cta_begin). A unit that
// spans several CTAs leaves partial (O, row max, row sum) records per query tile that a combine
// kernel merges with log-sum-exp weights.
//
// CTA roles (352 threads):
//   warps 0-3, 4-7  softmax warpgroup of query tile 0 / 1: thread r owns query row r (TMEM lane
//              r). Loads its Q tile into swizzled shared memory; per key tile reads S from TMEM,
//              masks unused page slots, takes the row max, then -- taking turns with the other
//              warpgroup, because the exponentials are the bottleneck (MUFU) -- computes
//              P = 2^(s*log2e/sqrt(D) - m) (FFMA + MUFU ex2), writes P as bf16 over the first
//              half of the same TMEM buffer and accumulates the row sum. O in TMEM is rescaled
//              only when the row max grows by more than 2^8 (lazy rescale).
//   warp 8     TMA producer: resolves the tile's 6 page ids and issues 12 page copies (K, V)
//              per tile into 4-stage K and V rings.
//   warps 9,10 MMA issuers, one per query tile: S(j) = Q K_j^T (A, B from shared memory) into
//              S/P buffer j % 2, then O += P(j-1) V_(j-1) with P read from TMEM (A operand in
//              tensor memory) and V from shared memory (MN-major).
// TMEM (512 columns): per query tile q, q*256 + {S/P buffer 0 [0,96), S/P buffer 1 [96,192),
// O fp32 [192,256)}. With two S/P buffers per query tile the softmax of tile j+1 never waits for
// P(j) V to finish: S(j+1) is computed into the other buffer while P(j) is still being read, and
// a buffer is reused only by the MMA issued after the P V that read it (tcgen05.mma operations
// of one thread execute in issue order).
// Every wait is bounded in time (AttnParams::wait_ns); on expiry the kernel sets
// GCA_DEVERR_WAIT_TIMEOUT and the CTA's abort flag, the producer waits (bounded) for the copies
// it issued, the MMA issuers wait (bounded) for the MMAs they issued, TMEM is freed and the
// kernel returns.
#include <cuda_bf16.h>

#include "gca_internal.h"

namespace gca {
namespace {

constexpr int kStages = 4;          // K and V rings
constexpr int kLensRing = 8;        // page-length words in flight (the producer leads the
                                    // softmax by at most kStages + 2 tiles)
constexpr int kSoftmaxWarps = 4 * kQPerCta;
constexpr int kThreads = 32 * (kSoftmaxWarps + 1 + kQPerCta);  // + TMA warp + MMA warps
constexpr int kWarpTma = kSoftmaxWarps;
constexpr int kWarpMma0 = kSoftmaxWarps + 1;  // MMA warp of query tile q: kWarpMma0 + q
constexpr uint32_t kQTileBytes = kTileQ * kHeadDim * 2;      // 16 KB
constexpr uint32_t kKvTileBytes = kTileK * kHeadDim * 2;     // 12 KB
constexpr uint32_t kPageBytes = kPageSize * kHeadDim * 2;    // 2 KB
constexpr uint64_t kFullLens = 0x0000101010101010ull;        // 6 pages of 16 valid slots
static_assert(kPagesPerTile == 6, "page-length word holds 6 pages");
// TMEM columns per query tile: two S/P buffers of kTileK columns, then O (64).
constexpr uint32_t kTmemPerQ = 256;
constexpr uint32_t kTmemCols = kTmemPerQ * kQPerCta;
constexpr uint32_t kColO = 2 * kTileK;
static_assert(kColO + kHeadDim == kTmemPerQ, "TMEM budget");
// Dynamic shared memory: query tiles, K ring, V ring (each tile 1024-byte aligned for the
// 128-byte swizzle), then the barrier block. No static shared memory, so the dynamic base is
// the start of the CTA's window (1024-aligned; checked at run time).
constexpr size_t kTilesBytes = (size_t)kQTileBytes * kQPerCta + (size_t)kKvTileBytes * 2 * kStages;
static_assert(kKvTileBytes % 1024 == 0 && kQTileBytes % 1024 == 0, "swizzle atoms");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows > 2^8

struct __align__(8) Shared {
  uint64_t k_full[kStages];
  uint64_t k_empty[kStages];
  uint64_t v_full[kStages];
  uint64_t v_empty[kStages];
  uint64_t lens_full[kLensRing];
  uint64_t lens[kLensRing];  // valid-slot count of each page of a tile, one byte per page
  uint64_t q_full[kQPerCta];
  uint64_t s_full[kQPerCta][2];   // S(j) of query tile q is in buffer j % 2
  uint64_t p_full[kQPerCta][2];   // P(j) of query tile q written over buffer j % 2
  uint64_t pv_done[kQPerCta][2];  // O += P(j) V_j of query tile q has completed
  uint64_t mma_drain[kQPerCta];   // every MMA of query tile q has completed (teardown)
  uint64_t turn[kQPerCta];        // exponential turns of the two softmax warpgroups
  uint32_t tmem_base;
  volatile int abort_flag;
};
constexpr size_t kSmemBytes = kTilesBytes + sizeof(Shared);

// ------------------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_addr(bar)),
      "r"(bytes)
      : "memory");
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Potentially blocking test: the thread may be suspended in hardware until the phase completes
// or a system-dependent time limit passes.
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, spinning (kSpin) or suspending in
// try_wait. Gives up when the CTA's abort flag is set (unless `drain`) or after p.wait_ns; a
// timeout sets the error bit and the abort flag.
template <bool kSpin>
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, Shared* sh,
                                           const AttnParams& p, bool drain = false) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (kSpin ? mbar_test(bar, parity) : mbar_try(bar, parity)) return true;
    if (!kSpin || (i & 63u) == 0u) {
      if (!drain && sh->abort_flag) return false;
      if (global_timer() - t0 > p.wait_ns) {
        sh->abort_flag = 1;
        atomicOr(p.err, GCA_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Every lane of the warp waits; the result is agreed across the warp so that warp-collective
// instructions after it never run with diverged lanes.
template <bool kSpin>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Shared* sh,
                                          const AttnParams& p, bool drain = false) {
  return __all_sync(0xffffffffu, wait_phase<kSpin>(bar, parity, sh, p, drain));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// The barrier's phase completes once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Loads of 32 lanes x 32 consecutive 32-bit TMEM columns into registers. tmem_ld_wait() must
// follow before the registers are used; the asm statements below are volatile and ordered, and
// the wait lists the loaded registers as read-write so no use is scheduled above it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Waits for this thread's outstanding TMEM loads; the 32 registers of each listed block are
// tied to the wait so that the compiler cannot read them before it.
template <int kBlocks>
__device__ __forceinline__ void tmem_ld_wait(float* v) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32 * kBlocks; ++i) asm volatile("" : "+f"(v[i]));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 descriptor version 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
  return (1u << 4)                      // D fp32
         | (1u << 7)                    // A bf16
         | (1u << 10)                   // B bf16
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(n >> 3) << 17)
         | ((uint32_t)(kTileQ >> 4) << 24);
}

// ------------------------------------------------------------------------- page walk

// Page ids of kBatchTiles consecutive steps, fetched in one round of loads: lane l <
// kBatchTiles * kPagesPerTile holds page l % kPagesPerTile of step s0 + l / kPagesPerTile (the
// logical pages of a key tile do not depend on the work unit, only on the tile index).
constexpr int kBatchTiles = 5;
static_assert(kBatchTiles * kPagesPerTile <= 32, "one page per lane");
struct PageBatch {
  int page, len;
};

__device__ __forceinline__ PageBatch fetch_pages(const AttnParams& p, int64_t s0, int64_t s_end,
                                                 int fallback, int lane) {
  PageBatch b{fallback, 0};
  const int64_t s = s0 + lane / kPagesPerTile;
  if (lane < kBatchTiles * kPagesPerTile && s < s_end) {
    const int j = (int)(s % p.n_tiles);
    resolve_page(p, j * kPagesPerTile + lane % kPagesPerTile, fallback, &b.page, &b.len);
  }
  return b;
}

// ------------------------------------------------------------------------- roles

// Warp 8: resolves each tile's pages and issues their K and V copies. The page ids are fetched
// kBatchTiles steps ahead of their use, so the page-table loads never stall the copies.
__device__ __forceinline__ void tma_producer(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                             const AttnParams& p, Shared& sh, uint8_t* k_smem,
                                             uint8_t* v_smem, int64_t s_begin, int64_t s_end) {
  const int lane = threadIdx.x & 31;
  int fallback = 0, flen = 0;
  resolve_page(p, 0, 0, &fallback, &flen);
  uint32_t it = 0;
  uint32_t issued_k = 0, issued_v = 0;  // tiles whose copies were issued (a prefix of it)
  bool ok = true;
  // test hook: CTA 0 never issues the copies of its first tile, so the MMA issuer's wait for
  // them runs out (nothing is in flight for that tile at any time)
  const bool withhold_first = p.withhold != 0 && blockIdx.x == 0;
  PageBatch cur = fetch_pages(p, s_begin, s_end, fallback, lane);
  PageBatch nxt = fetch_pages(p, s_begin + kBatchTiles, s_end, fallback, lane);
  for (int64_t s = s_begin; s < s_end && ok;) {
    const int u2 = (int)(s / p.n_tiles);
    const int64_t seg_end = min(s_end, (int64_t)(u2 + 1) * p.n_tiles);
    const int h = u2 / p.n_pairs;
    const int j_end = (int)(seg_end - (int64_t)u2 * p.n_tiles);
    for (int j = (int)(s - (int64_t)u2 * p.n_tiles); j < j_end; ++j, ++it) {
      const int st = it % kStages;
      const uint32_t use = it / kStages;
      const int kb = (int)(it % kBatchTiles);
      if (kb == 0 && it > 0) {
        cur = nxt;
        nxt = fetch_pages(p, s_begin + it + kBatchTiles, s_end, fallback, lane);
      }
      int page = __shfl_sync(0xffffffffu, cur.page, kb * kPagesPerTile + lane % kPagesPerTile);
      int len = __shfl_sync(0xffffffffu, cur.len, kb * kPagesPerTile + lane % kPagesPerTile);
      if (lane < kPagesPerTile && (page < 0 || page >= p.num_pages)) {
        atomicOr(p.err, GCA_DEVERR_PAGE_RANGE);
        page = 0;
        len = 0;
      }
      uint64_t lens = 0;
#pragma unroll
      for (int k = 0; k < kPagesPerTile; ++k) {
        lens |= (uint64_t)(uint32_t)__shfl_sync(0xffffffffu, len, k) << (8 * k);
      }
      const int row = (page * p.H + h) * kPageSize;
      if (use > 0 && !warp_wait<false>(&sh.k_empty[st], (use - 1) & 1u, &sh, p)) {
        ok = false;
        break;
      }
      if (withhold_first && it == 0) {
        if (lane == 0) {
          sh.lens[it % kLensRing] = lens;
          mbar_arrive(&sh.lens_full[it % kLensRing]);
        }
        __syncwarp();
        ok = false;  // nothing more is issued; the waits downstream run out
        break;
      }
      if (lane == 0) {
        sh.lens[it % kLensRing] = lens;
        mbar_arrive(&sh.lens_full[it % kLensRing]);
        mbar_arrive_expect_tx(&sh.k_full[st], kKvTileBytes);
      }
      __syncwarp();
      if (lane < kPagesPerTile) {
        tma_load_2d(smem_addr(k_smem + st * kKvTileBytes + lane * kPageBytes), tm_k, 0, row,
                    &sh.k_full[st]);
      }
      issued_k = it + 1;
      if (use > 0 && !warp_wait<false>(&sh.v_empty[st], (use - 1) & 1u, &sh, p)) {
        ok = false;
        break;
      }
      if (lane == 0) mbar_arrive_expect_tx(&sh.v_full[st], kKvTileBytes);
      __syncwarp();
      if (lane < kPagesPerTile) {
        tma_load_2d(smem_addr(v_smem + st * kKvTileBytes + lane * kPageBytes), tm_v, 0, row,
                    &sh.v_full[st]);
      }
      issued_v = it + 1;
    }
    s = seg_end;
  }
  // Drain: wait until the copies issued last have landed before the CTA can exit (a stage is
  // reissued only after its previous copy was consumed, so only the last kStages can be live).
  for (uint32_t q = issued_k > (uint32_t)kStages ? issued_k - kStages : 0u; q < issued_k; ++q) {
    warp_wait<false>(&sh.k_full[q % kStages], (q / kStages) & 1u, &sh, p, true);
  }
  for (uint32_t q = issued_v > (uint32_t)kStages ? issued_v - kStages : 0u; q < issued_v; ++q) {
    warp_wait<false>(&sh.v_full[q % kStages], (q / kStages) & 1u, &sh, p, true);
  }
}

// Warps 9 and 10, one elected thread each: the MMAs of query tile qq.
__device__ __forceinline__ void mma_issuer(const AttnParams& p, Shared& sh, uint32_t tmem,
                                           uint8_t* q_smem, uint8_t* k_smem, uint8_t* v_smem,
                                           int qq, int64_t s_begin, int64_t s_end) {
  constexpr uint32_t kIdescS = idesc_bf16(kTileK, false);
  constexpr uint32_t kIdescPV = idesc_bf16(kHeadDim, true);
  const uint32_t tq = tmem + kTmemPerQ * qq;
  const uint64_t q_desc = sw128_desc(smem_addr(q_smem + qq * kQTileBytes), 16, 1024);
  uint32_t it = 0, seg = 0;
  bool ok = true;
  for (int64_t s = s_begin; s < s_end && ok; ++seg) {
    const int u2 = (int)(s / p.n_tiles);
    const int64_t seg_end = min(s_end, (int64_t)(u2 + 1) * p.n_tiles);
    const int n = (int)(seg_end - s);
    if (!wait_phase<true>(&sh.q_full[qq], seg & 1u, &sh, p)) break;
    tc_fence_after();
    for (int i = 0; i <= n; ++i) {
      if (i < n) {  // S(it + i) = Q K^T into buffer (it + i) % 2
        const uint32_t cur = it + i;
        const int st = cur % kStages;
        if (!wait_phase<true>(&sh.k_full[st], (cur / kStages) & 1u, &sh, p)) { ok = false; break; }
        tc_fence_after();
        const uint64_t k_desc = sw128_desc(smem_addr(k_smem + st * kKvTileBytes), 16, 1024);
        const uint32_t d = tq + (cur & 1u) * kTileK;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          // +32 bytes along K inside the swizzled 128-byte rows
          mma_ss(d, q_desc + 2 * kk, k_desc + 2 * kk, kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sh.s_full[qq][cur & 1u]);
        mma_commit(&sh.k_empty[st]);
      }
      if (i > 0) {  // O += P(it + i - 1) V
        const uint32_t prv = it + i - 1;
        const int st = prv % kStages;
        if (!wait_phase<true>(&sh.p_full[qq][prv & 1u], (prv >> 1) & 1u, &sh, p)) { ok = false; break; }
        if (!wait_phase<true>(&sh.v_full[st], (prv / kStages) & 1u, &sh, p)) { ok = false; break; }
        tc_fence_after();
        const uint64_t v_desc = sw128_desc(smem_addr(v_smem + st * kKvTileBytes), 16384, 1024);
        const uint32_t a = tq + (prv & 1u) * kTileK;
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk) {
          // 16 keys: 2048 bytes of V, 8 TMEM columns of packed P
          mma_ts(tq + kColO, a + 8 * kk, v_desc + 128 * kk, kIdescPV,
                 (i > 1 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh.pv_done[qq][prv & 1u]);
        mma_commit(&sh.v_empty[st]);
      }
    }
    it += n;
    s = seg_end;
  }
  // Teardown: TMEM may be freed only once every MMA issued here has completed.
  mma_commit(&sh.mma_drain[qq]);
  wait_phase<true>(&sh.mma_drain[qq], 0u, &sh, p, true);
}

// Warpgroup qq (warps 4*qq .. 4*qq+3): softmax of query tile qq; thread r owns row r.
__device__ __forceinline__ void softmax_group(const AttnParams& p, Shared& sh, uint32_t tmem,
                                              uint8_t* q_smem, int64_t s_begin, int64_t s_end) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qq = warp >> 2;
  const int r = (warp & 3) * 32 + lane;
  const uint32_t t_row = tmem + kTmemPerQ * qq + ((uint32_t)((warp & 3) * 32) << 16);
  uint8_t* q_tile = q_smem + qq * kQTileBytes;
  uint32_t it = 0, turns = 0;
  uint32_t n_exact = 0, n_rescale = 0;  // branch counts of this row (past each first tile)
  bool ok = true;
  // The two warpgroups take turns for the exponentials (MUFU-bound): while one computes them,
  // the other waits for its next S, loads it and reduces the row max, so the two stay half a
  // tile apart instead of stalling on their loads at the same time. Query tile 0 goes first.
  uint64_t* const my_turn = &sh.turn[qq];
  uint64_t* const their_turn = &sh.turn[qq ^ 1];
  if (qq == 1) mbar_arrive(their_turn);
  for (int64_t s = s_begin; s < s_end && ok;) {
    const int u2 = (int)(s / p.n_tiles);
    const int64_t seg_end = min(s_end, (int64_t)(u2 + 1) * p.n_tiles);
    const int j0 = (int)(s - (int64_t)u2 * p.n_tiles);
    const int j1 = (int)(seg_end - (int64_t)u2 * p.n_tiles);
    const int h = u2 / p.n_pairs;
    const int qt = (u2 % p.n_pairs) * kQPerCta + qq;
    const int qi = qt * kTileQ + r;

    // Q row -> shared memory, 128-byte swizzle (16-byte chunk c of row r at c ^ (r % 8)),
    // and its squared norm. The previous segment's MMAs that read this tile have completed
    // (its epilogue waited for the last P V, issued after every S of the segment).
    float q2 = 0.f;
    {
      const bool valid = qt < p.n_qt && qi < p.T;
      const uint4* src = p.q + ((int64_t)qi * p.H + h) * 8;
      uint8_t* row = q_tile + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v = valid ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = v;
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float a = __uint_as_float(vw[w] << 16), b = __uint_as_float(vw[w] & 0xffff0000u);
          q2 = fmaf(a, a, fmaf(b, b, q2));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&sh.q_full[qq]);
    }
    // Every score of this row is at most |q| * max|k| (Cauchy-Schwarz; max|k| over every key
    // appended to the cache, so it covers the keys this row sees). While that bound is within
    // the lazy-rescale threshold of the running max, a tile's exact max cannot trigger a
    // rescale, so the max pass is skipped and the same branch is taken. The factor covers
    // rounding in the norms (a bound a hair too small only lets P reach 2^8 * (1 + eps)).
    const float score_bound = sqrtf(q2 * __uint_as_float(p.kmax[h])) * 1.01f * p.scale_log2;

    float m_run = -INFINITY;  // running row max, log2 units (scaled)
    float l_run = 0.f;        // running row sum relative to m_run
    for (int j = j0; j < j1; ++j, ++it) {
      const uint32_t b = it & 1u;
      if (!warp_wait<false>(&sh.s_full[qq][b], (it >> 1) & 1u, &sh, p)) { ok = false; break; }
      if (!warp_wait<false>(&sh.lens_full[it % kLensRing], (it / kLensRing) & 1u, &sh, p)) {
        ok = false;
        break;
      }
      const uint64_t lens = sh.lens[it % kLensRing];
      tc_fence_after();
      const uint32_t t_buf = t_row + b * kTileK;
      float sv[kTileK];
      tmem_ld32(t_buf + 0, sv);
      tmem_ld32(t_buf + 32, sv + 32);
      tmem_ld32(t_buf + 64, sv + 64);
      tmem_ld_wait<3>(sv);

      if (lens != kFullLens) {
#pragma unroll
        for (int pg = 0; pg < kPagesPerTile; ++pg) {
          const int len = (int)((lens >> (8 * pg)) & 0xffu);
          if (len < kPageSize) {
#pragma unroll
            for (int c = 0; c < kPageSize; ++c) {
              if (c >= len) sv[pg * kPageSize + c] = -INFINITY;
            }
          }
        }
      }
      float m_new = m_run, alpha = 1.f;
      if (!(score_bound <= m_run + kRescaleThreshold)) {
        // row max: 8 independent chains of 3-input max
        float mx[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmaxf(sv[2 * a], sv[2 * a + 1]);
#pragma unroll
        for (int c = 16; c < kTileK; c += 16) {
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = max3(mx[a], sv[c + 2 * a], sv[c + 2 * a + 1]);
        }
#pragma unroll
        for (int w = 4; w >= 1; w /= 2) {
#pragma unroll
          for (int a = 0; a < w; ++a) mx[a] = fmaxf(mx[a], mx[a + w]);
        }
        const float tile_max = mx[0] * p.scale_log2;
        if (tile_max > m_run + kRescaleThreshold) {
          m_new = tile_max;
          alpha = ex2(m_run - m_new);
          n_rescale += j > j0 ? 1u : 0u;
        }
        n_exact += j > j0 ? 1u : 0u;
      }
      // Lazy rescale of O (rare): O += P(j-1) V must have completed first; P(j) V is issued
      // only after this thread's p_full arrival below.
      if (j > j0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        const uint32_t pb = (it - 1) & 1u;
        if (!warp_wait<false>(&sh.pv_done[qq][pb], ((it - 1) >> 1) & 1u, &sh, p)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kHeadDim / 16; ++c) {
          float o[16];
          tmem_ld16(t_row + kColO + 16 * c, o);
#pragma unroll
          for (int a = 0; a < 16; ++a) o[a] *= alpha;
          tmem_st16(t_row + kColO + 16 * c, o);
        }
      }
      // P = 2^(s*c - m), in this warpgroup's turn: scale-subtract, exponentials, bf16
      // packing, row sum; P goes to the first 48 columns of the buffer S came from (S is dead
      // once loaded). The turn passes to the other warpgroup one 32-column chunk before the
      // end, so that its first exponentials queue behind this group's last ones.
      if (!warp_wait<true>(my_turn, turns & 1u, &sh, p)) { ok = false; break; }
      ++turns;
      const float neg_m = -m_new;
#pragma unroll
      for (int e = 0; e < kTileK; ++e) sv[e] = fmaf(sv[e], p.scale_log2, neg_m);
      float rs[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) rs[a] = 0.f;
#pragma unroll
      for (int chunk = 0; chunk < kTileK / 32; ++chunk) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = 32 * chunk + 2 * c;
          const float e0 = ex2(sv[e]);
          const float e1 = ex2(sv[e + 1]);
          pk[c] = pack_bf2(e0, e1);
          rs[2 * (c & 3)] += e0;
          rs[2 * (c & 3) + 1] += e1;
        }
        tmem_st16(t_buf + 16 * chunk, reinterpret_cast<const float*>(pk));
        if (chunk == kTileK / 32 - 2) mbar_arrive(their_turn);
      }
      const float row_sum =
          ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      l_run = l_run * alpha + row_sum;
      m_run = m_new;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.p_full[qq][b]);
    }
    if (!ok) break;

    // ---- epilogue: the last P V of the segment has completed
    {
      const uint32_t lb = (it - 1) & 1u;
      if (!warp_wait<false>(&sh.pv_done[qq][lb], ((it - 1) >> 1) & 1u, &sh, p)) break;
    }
    tc_fence_after();
    float o[kHeadDim];
    tmem_ld32(t_row + kColO, o);
    tmem_ld32(t_row + kColO + 32, o + 32);
    tmem_ld_wait<2>(o);
    tc_fence_before();
    if (qt < p.n_qt) {
      if (j0 == 0 && j1 == p.n_tiles) {
        if (qi < p.T) {
          const float inv = 1.f / l_run;
          uint4* dst = p.out + ((int64_t)qi * p.H + h) * 8;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 w;
            w.x = pack_bf2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
            w.y = pack_bf2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
            w.z = pack_bf2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
            w.w = pack_bf2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
            dst[c] = w;
          }
        }
      } else {
        const int64_t slot = part_slot(blockIdx.x, u2, qq);
        float4* dst = reinterpret_cast<float4*>(p.part_o + (slot * kTileQ + r) * kHeadDim);
#pragma unroll
        for (int c = 0; c < kHeadDim / 4; ++c) {
          dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
        p.part_ml[slot * kTileQ + r] = make_float2(m_run, l_run);
      }
    }
    s = seg_end;
  }
  // one atomic per warp and counter, at the end
  const uint32_t we = __reduce_add_sync(0xffffffffu, n_exact);
  const uint32_t wr = __reduce_add_sync(0xffffffffu, n_rescale);
  if (lane == 0 && we != 0u) atomicAdd(&p.counters[0], (unsigned long long)we);
  if (lane == 0 && wr != 0u) atomicAdd(&p.counters[1], (unsigned long long)wr);
}

// ------------------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_addr(smem) & 1023u) != 0u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(p.err, GCA_DEVERR_SMEM_ALIGN);
    return;
  }
  Shared& sh = *reinterpret_cast<Shared*>(smem + kTilesBytes);
  uint8_t* q_smem = smem;                                      // kQPerCta query tiles
  uint8_t* k_smem = smem + kQPerCta * kQTileBytes;             // kStages key tiles
  uint8_t* v_smem = k_smem + kStages * kKvTileBytes;           // kStages value tiles
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.k_full[s], 1);
      mbar_init(&sh.k_empty[s], kQPerCta);
      mbar_init(&sh.v_full[s], 1);
      mbar_init(&sh.v_empty[s], kQPerCta);
    }
    for (int s = 0; s < kLensRing; ++s) mbar_init(&sh.lens_full[s], 1);
    for (int q = 0; q < kQPerCta; ++q) {
      mbar_init(&sh.q_full[q], kTileQ);
      mbar_init(&sh.mma_drain[q], 1);
      mbar_init(&sh.turn[q], kTileQ);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sh.s_full[q][b], 1);
        mbar_init(&sh.p_full[q][b], kTileQ);
        mbar_init(&sh.pv_done[q][b], 1);
      }
    }
    sh.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma0) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
            smem_addr(&sh.tmem_base)),
        "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // Everything above is local (barriers, TMEM); from here on the kernel reads the page table,
  // Q, K and V that earlier work in the stream wrote.
  pdl_wait();

  // A cache whose sticky error word is set gets no further work: every role sees an empty step
  // range and the CTA goes straight to its teardown.
  const bool dead = *reinterpret_cast<volatile uint32_t*>(p.err) != 0u;
  const int64_t s_begin = cta_begin(blockIdx.x, p);
  const int64_t s_end = dead ? s_begin : cta_begin(blockIdx.x + 1, p);

  if (warp == kWarpTma) {
    tma_producer(&tm_k, &tm_v, p, sh, k_smem, v_smem, s_begin, s_end);
  } else if (warp == kWarpMma0 || warp == kWarpMma0 + 1) {
    if ((threadIdx.x & 31) == 0) {
      mma_issuer(p, sh, tmem, q_smem, k_smem, v_smem, warp - kWarpMma0, s_begin, s_end);
    }
    __syncwarp();
  } else {
    softmax_group(p, sh, tmem, q_smem, s_begin, s_end);
  }

  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

}  // namespace

cudaError_t attn_prepare(int* ctas_per_sm) {
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  // One CTA per SM: it holds all 512 TMEM columns (two query tiles).
  *ctas_per_sm = 1;
  return cudaSuccess;
}

cudaError_t launch_attn(const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                        cudaStream_t s) {
  return launch_dependent(attn_kernel, dim3(p.grid), dim3(kThreads), kSmemBytes, s, tk, tv, p);
}

}  // namespace gca
