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
// the page table. A 128-key tile is 8 pages; each page of one head is a contiguous 2 KB block
// [16 slots][64 dims] bf16 that TMA copies into shared memory with the 128-byte swizzle.
//
// Work split: a CTA works on two 128-query tiles of one head at once (they see the same keys,
// so every K/V tile is fetched once for both); a (head, tile pair) is a work unit. The flattened
// (unit, key tile) steps are cut into `grid` equal ranges, one per CTA (one CTA per SM). A unit
// that spans several CTAs leaves partial (O, row max, row sum) records per query tile that a
// combine kernel merges with log-sum-exp weights.
//
// CTA roles (352 threads):
//   warps 0-3, 4-7  softmax warpgroup of query tile 0 / 1: thread r owns query row r (TMEM lane
//              r). Loads its Q tile into swizzled shared memory; per key tile reads S from TMEM,
//              masks unused page slots, takes the row max, then -- taking turns with the other
//              warpgroup, because the exponentials are the bottleneck (MUFU) -- computes
//              P = 2^(s*log2e/sqrt(D) - m), writes it to TMEM as bf16 and accumulates the row
//              sum; O in TMEM is rescaled only when the row max grows by more than 2^8.
//   warp 8     TMA producer: resolves the tile's 8 page ids and issues 16 page copies (K, V)
//              per tile into 3-stage K and V rings.
//   warps 9,10 MMA issuers, one per query tile (one thread issues only about one tcgen05.mma
//              per 60 cycles): S = Q K^T (A, B from shared memory) into TMEM, then O += P V with
//              P read from TMEM (A operand in tensor memory) and V from shared memory (MN-major).
//              S of tile j+1 is issued as soon as S of tile j has been read.
// TMEM (512 columns): per query tile q, q*256 + {S fp32 [0,128), P bf16x2 [128,192),
// O fp32 [192,256)}.
// Every wait is bounded in time; on expiry the kernel sets GCA_DEVERR_WAIT_TIMEOUT, drains its
// own copies, frees TMEM and returns.
#include <cuda_bf16.h>

#include "gca_internal.h"

// Build options (defaults are the fastest measured on B200 at head_dim 64):
//   GCA_MAX_CHAINS independent 3-input max chains for the row max.
//   GCA_SLEEP_WAIT 1: barrier waits suspend the thread in hardware (try_wait with a suspend
//                  time hint) instead of spinning on issue slots.
#ifndef GCA_MAX_CHAINS
#define GCA_MAX_CHAINS 8
#endif
#ifndef GCA_SLEEP_WAIT
#define GCA_SLEEP_WAIT 1
#endif
//   GCA_TURN_SPIN  0: the exponential-turn wait sleeps in hardware; 1: it spins; n >= 2: it
//                  spins with __nanosleep(n) between polls.
//   GCA_TURN_EARLY the turn passes to the other warpgroup this many 32-column chunks before
//                  this one's exponentials are done.
//   GCA_MMA_SPIN   1: the MMA-issuing threads spin on their barriers; 0: they sleep in try_wait.
#ifndef GCA_MMA_SPIN
#define GCA_MMA_SPIN 1
#endif
//   GCA_TURNS      1: the two softmax warpgroups take turns for the exponentials; 0: both
//                  compute them whenever their scores are ready.
#ifndef GCA_TURNS
#define GCA_TURNS 1
#endif
#ifndef GCA_TURN_SPIN
#define GCA_TURN_SPIN 1
#endif
#ifndef GCA_TURN_EARLY
#define GCA_TURN_EARLY 1
#endif
//   GCA_POLY_PAIRS of every 16 pairs of exponentials, this many are computed on the FMA pipe
//                  with a cubic polynomial instead of MUFU (relieves the MUFU bottleneck).
#ifndef GCA_POLY_PAIRS
#define GCA_POLY_PAIRS 0
#endif
//   GCA_F32X2      1: the scale-subtract and the row sum use packed f32x2 FMA / add (half the
//                  instructions of the scalar forms).
#ifndef GCA_F32X2
#define GCA_F32X2 0
#endif
//   GCA_FFMA_CHUNK 1: the scale-subtract runs per 32-column chunk, just before its exponentials.
#ifndef GCA_FFMA_CHUNK
#define GCA_FFMA_CHUNK 0
#endif
//   GCA_TURN_WARP  1: the turn alternates per SM sub-partition: warp w of one warpgroup hands
//                  it to warp w of the other (the two share that sub-partition's MUFU); 0: the
//                  whole warpgroup hands over at once (waits for its slowest warp).
#ifndef GCA_TURN_WARP
#define GCA_TURN_WARP 0
#endif

#ifndef GCA_TRACE
#define GCA_TRACE 0
#endif

namespace gca {

#if GCA_TRACE
// Event timestamps (clock64) of the first tiles of CTAs 0 and 1, for pipeline studies; read
// back with gca_debug_trace in builds with -DGCA_TRACE=1.
__device__ long long g_trace[2][64][32];
#define TRACE(slot, tile)                                                                   \
  do {                                                                                      \
    if (blockIdx.x < 2 && (tile) < 64) g_trace[blockIdx.x][(tile)][(slot)] = clock64();     \
  } while (0)
#else
#define TRACE(slot, tile) \
  do {                    \
  } while (0)
#endif

namespace {

constexpr int kKStages = 3;        // K ring: a slot frees once both S = Q K^T are computed
constexpr int kVStages = 3;        // V ring: a slot frees after both O += P V
constexpr int kSoftmaxWarps = 4 * kQPerCta;
constexpr int kThreads = 32 * (kSoftmaxWarps + 1 + kQPerCta);  // + TMA warp + MMA warps
constexpr int kWarpTma = kSoftmaxWarps;
constexpr int kWarpMma0 = kSoftmaxWarps + 1;  // MMA warp of query tile q: kWarpMma0 + q
constexpr uint32_t kTileBytes = kTileK * kHeadDim * 2;      // 16 KB
constexpr uint32_t kPageBytes = kPageSize * kHeadDim * 2;    // 2 KB
// TMEM: per query tile q, columns q*256 + {S fp32 [0,128), P bf16x2 [128,192), O fp32 [192,256)}.
constexpr uint32_t kTmemPerQ = 256;
constexpr uint32_t kTmemCols = kTmemPerQ * kQPerCta;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;
// Dynamic shared memory: query tiles, K ring, V ring (each tile 1024-byte aligned for the
// 128-byte swizzle), then the barrier block. No static shared memory, so the dynamic base is
// the start of the CTA's window (1024-aligned; checked at run time).
constexpr size_t kTilesBytes = (size_t)kTileBytes * (kQPerCta + kKStages + kVStages);
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale O when the max grows > 2^8

struct __align__(8) Shared {
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  // Valid-slot counts (one byte per page) of tile it live in lens[it % 4], published through
  // lens_full[it % 4]; the producer cannot get 4 tiles ahead of the softmax warps because it
  // waits for the V slot of tile it-3 (freed after P(it-3) V) before issuing tile it+1.
  uint64_t lens_full[4];
  uint64_t lens[4];
  uint64_t q_full[kQPerCta];
  uint64_t s_full[kQPerCta];
  uint64_t s_free[kQPerCta];
  uint64_t p_full[kQPerCta];
  uint64_t pv_done[kQPerCta];
  uint64_t turn[kQPerCta][4];  // exponential turns of the two softmax warpgroups (per warp
                               // when GCA_TURN_WARP, else [q][0] for the whole warpgroup)
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

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
#if GCA_SLEEP_WAIT
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
      : "memory");
#else
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
#endif
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Gives up when the CTA's abort flag is
// set (unless `drain`) or after kWaitNs; a timeout sets the error bit and the abort flag.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, Shared* sh,
                                        uint32_t* err, bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (GCA_SLEEP_WAIT || (i & 63u) == 0u) {
      if (!drain && sh->abort_flag) return false;
      if (global_timer() - t0 > kWaitNs) {
        sh->abort_flag = 1;
        atomicOr(err, GCA_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Spinning variant (no hardware suspend) for short, latency-critical hand-overs: a thread
// suspended in try_wait resumes some hundreds of cycles after the phase completes.
template <int kBackoffNs = 0>
__device__ __forceinline__ bool spin_phase(uint64_t* bar, uint32_t parity, Shared* sh,
                                           uint32_t* err) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (kBackoffNs > 0) __nanosleep(kBackoffNs);
    if (mbar_test_wait(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (sh->abort_flag) return false;
      if (global_timer() - t0 > kWaitNs) {
        sh->abort_flag = 1;
        atomicOr(err, GCA_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// The MMA issuers' waits: on the critical path from "P ready" to "P V issued".
__device__ __forceinline__ bool mma_wait(uint64_t* bar, uint32_t parity, Shared* sh,
                                         uint32_t* err) {
#if GCA_MMA_SPIN
  return spin_phase(bar, parity, sh, err);
#else
  return wait_phase(bar, parity, sh, err);
#endif
}

// Every lane of the warp waits; the result is agreed across the warp so that warp-collective
// instructions after it never run with diverged lanes.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Shared* sh,
                                          uint32_t* err, bool drain = false) {
  return __all_sync(0xffffffffu, wait_phase(bar, parity, sh, err, drain));
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

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Loads of 32 lanes x N consecutive 32-bit TMEM columns into registers, each followed by
// tcgen05.wait::ld inside the same asm statement, so the compiler cannot schedule a use of the
// registers before the data has arrived.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%129];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95}, [%130];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%131];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr + 0u), "r"(taddr + 32u), "r"(taddr + 64u), "r"(taddr + 96u)
      : "memory");
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr + 0u), "r"(taddr + 32u)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr + 0u)
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

// 2^x on the FMA pipe. Range reduction x = j + r, j = round(x) (adding 1.5 * 2^23 leaves j in
// the low mantissa bits), r in [-1/2, 1/2]; 2^r from a cubic fitted here for least maximum
// relative error on [-1/2, 1/2] (Lawson-reweighted least squares); 2^j joins by an integer add
// into the exponent field. Max relative error 7.5e-5 (float32), far below the bf16 rounding
// of P that follows. x is clamped at -125 so the exponent add stays in range (masked -inf
// scores give 2^-125 instead of 0).
__device__ __forceinline__ float exp2_poly(float x) {
  constexpr float kMagic = 12582912.0f;
  constexpr float kC0 = 0.9999281167984009f, kC1 = 0.6932609677314758f;
  constexpr float kC2 = 0.24261054396629333f, kC3 = 0.05517132207751274f;
  x = fmaxf(x, -125.0f);
  const float t = x + kMagic;
  const float r = x - (t - kMagic);
  float q = fmaf(kC3, r, kC2);
  q = fmaf(q, r, kC1);
  q = fmaf(q, r, kC0);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

#if GCA_F32X2
// x = x * c + b on a pair (packed f32x2 FMA).
__device__ __forceinline__ void fma2_pair(float& x0, float& x1, float c, float b) {
  asm("{\n\t.reg .b64 x, cc, bb;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 cc, {%2, %2};\n\t"
      "mov.b64 bb, {%3, %3};\n\tfma.rn.f32x2 x, x, cc, bb;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(c), "f"(b));
}

// (a0, a1) += (b0, b1) (packed f32x2 add).
__device__ __forceinline__ void add2_pair(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 a, a, b;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
#endif

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

// Physical page and valid-slot count of logical page lp (anchor, window, trajectory order).
__device__ __forceinline__ void resolve_page(const AttnParams& p, int lp, int fallback,
                                             int* page, int* len) {
  if (lp < p.na_pages) {
    *page = p.frame_pages[lp];
    *len = (lp % p.ppf == p.ppf - 1) ? p.last_len : kPageSize;
  } else if (lp < p.na_pages + p.nw_pages) {
    const int w = lp - p.na_pages;
    *page = p.frame_pages[p.win_base + w];
    *len = (w % p.ppf == p.ppf - 1) ? p.last_len : kPageSize;
  } else if (lp < p.n_lp) {
    const int tp = lp - p.na_pages - p.nw_pages;
    *page = p.traj_pages[tp];
    *len = (tp == p.n_traj_pages - 1) ? p.traj_tail_len : kPageSize;
  } else {
    *page = fallback;  // any visible page: finite data, fully masked
    *len = 0;
  }
}

// ------------------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_signal_early();
  if ((smem_addr(smem) & 1023u) != 0u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(p.err, GCA_DEVERR_SMEM_ALIGN);
    return;
  }
  Shared& sh = *reinterpret_cast<Shared*>(smem + kTilesBytes);
  uint8_t* q_smem = smem;                                   // kQPerCta query tiles
  uint8_t* k_smem = smem + kQPerCta * kTileBytes;           // kKStages key tiles
  uint8_t* v_smem = k_smem + kKStages * kTileBytes;         // kVStages value tiles

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sh.k_full[s], 1);
      mbar_init(&sh.k_empty[s], kQPerCta);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sh.v_full[s], 1);
      mbar_init(&sh.v_empty[s], kQPerCta);
    }
    for (int s = 0; s < 4; ++s) mbar_init(&sh.lens_full[s], 1);
    for (int q = 0; q < kQPerCta; ++q) {
      mbar_init(&sh.q_full[q], kTileQ);
      mbar_init(&sh.s_full[q], 1);
      mbar_init(&sh.s_free[q], kTileQ);
      mbar_init(&sh.p_full[q], kTileQ);
      mbar_init(&sh.pv_done[q], 1);
      for (int w = 0; w < 4; ++w) mbar_init(&sh.turn[q][w], GCA_TURN_WARP ? 1 : kTileQ);
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
  const int64_t s_begin = (int64_t)blockIdx.x * p.total / p.grid;
  const int64_t s_end = dead ? s_begin : (int64_t)(blockIdx.x + 1) * p.total / p.grid;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    int fallback = 0;
    int flen = 0;
    resolve_page(p, 0, 0, &fallback, &flen);
    uint32_t it = 0, nk = 0, nv = 0;  // tiles walked; K and V copies issued
    bool ok = true;
    for (int64_t s = s_begin; s < s_end && ok;) {
      const int u2 = (int)(s / p.n_tiles);
      const int64_t seg_end = min(s_end, (int64_t)(u2 + 1) * p.n_tiles);
      const int h = u2 / p.n_pairs;
      for (int j = (int)(s - (int64_t)u2 * p.n_tiles); j < (int)(seg_end - (int64_t)u2 * p.n_tiles);
           ++j, ++it) {
        const int ks = it % kKStages, vs = it % kVStages;
        const uint32_t kuse = it / kKStages, vuse = it / kVStages;
        int page = 0, len = 0;
        if (lane < kPagesPerTile) resolve_page(p, j * kPagesPerTile + lane, fallback, &page, &len);
        if (page < 0 || page >= p.num_pages) {
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
        if (kuse > 0 && !warp_wait(&sh.k_empty[ks], (kuse - 1) & 1u, &sh, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          TRACE(0, it);
          sh.lens[it & 3] = lens;
          mbar_arrive(&sh.lens_full[it & 3]);
          mbar_arrive_expect_tx(&sh.k_full[ks], kTileBytes);
        }
        __syncwarp();
        if (lane < kPagesPerTile) {
          tma_load_2d(smem_addr(k_smem + ks * kTileBytes + lane * kPageBytes), &tm_k, 0, row,
                      &sh.k_full[ks]);
        }
        ++nk;
        if (vuse > 0 && !warp_wait(&sh.v_empty[vs], (vuse - 1) & 1u, &sh, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          TRACE(1, it);
          mbar_arrive_expect_tx(&sh.v_full[vs], kTileBytes);
        }
        __syncwarp();
        if (lane < kPagesPerTile) {
          tma_load_2d(smem_addr(v_smem + vs * kTileBytes + lane * kPageBytes), &tm_v, 0, row,
                      &sh.v_full[vs]);
        }
        ++nv;
      }
      s = seg_end;
    }
    // Drain: wait until the copies issued last have landed before the CTA can exit.
    for (uint32_t q = nk > (uint32_t)kKStages ? nk - kKStages : 0u; q < nk; ++q) {
      warp_wait(&sh.k_full[q % kKStages], (q / kKStages) & 1u, &sh, p.err, true);
    }
    for (uint32_t q = nv > (uint32_t)kVStages ? nv - kVStages : 0u; q < nv; ++q) {
      warp_wait(&sh.v_full[q % kVStages], (q / kVStages) & 1u, &sh, p.err, true);
    }
  } else if (warp == kWarpMma0 || warp == kWarpMma0 + 1) {
    // ------------------------------------------------------------ MMA issuers, one per query
    // tile (a thread issues about one tcgen05.mma per 60 cycles, so one thread could not keep
    // the tensor core fed for both tiles). Per key tile j: S(j) = Q K_j^T as soon as the
    // softmax warps have read S(j-1); then O += P(j-1) V_(j-1).
    const int qq = warp - kWarpMma0;
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kTileK, false);
      constexpr uint32_t kIdescPV = idesc_bf16(kHeadDim, true);
      const uint32_t tq = tmem + kTmemPerQ * qq;
      const uint64_t q_desc = sw128_desc(smem_addr(q_smem + qq * kTileBytes), 16, 1024);
      uint32_t it = 0, seg = 0;
      bool ok = true;
      for (int64_t s = s_begin; s < s_end && ok; ++seg) {
        const int u2 = (int)(s / p.n_tiles);
        const int64_t seg_end = min(s_end, (int64_t)(u2 + 1) * p.n_tiles);
        const int j0 = (int)(s - (int64_t)u2 * p.n_tiles);
        const int j1 = (int)(seg_end - (int64_t)u2 * p.n_tiles);
        if (!wait_phase(&sh.q_full[qq], seg & 1u, &sh, p.err)) break;
        tc_fence_after();
        for (int j = j0; j <= j1; ++j) {
          if (j < j1) {
            const int ks = it % kKStages;
            if (!mma_wait(&sh.k_full[ks], (it / kKStages) & 1u, &sh, p.err)) { ok = false; break; }
            if (j > j0 && !mma_wait(&sh.s_free[qq], (it - 1) & 1u, &sh, p.err)) { ok = false; break; }
            tc_fence_after();
            TRACE(qq ? 20 : 2, it);
            const uint64_t k_desc = sw128_desc(smem_addr(k_smem + ks * kTileBytes), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk) {
              // +32 bytes along K inside the swizzled 128-byte rows
              mma_ss(tq + kColS, q_desc + 2 * kk, k_desc + 2 * kk, kIdescS, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sh.s_full[qq]);
            mma_commit(&sh.k_empty[ks]);
            TRACE(qq ? 21 : 3, it);
          }
          if (j > j0) {
            const uint32_t pit = it - 1;  // tile j-1
            const int vs = pit % kVStages;
            if (!mma_wait(&sh.p_full[qq], pit & 1u, &sh, p.err)) { ok = false; break; }
            if (!mma_wait(&sh.v_full[vs], (pit / kVStages) & 1u, &sh, p.err)) { ok = false; break; }
            tc_fence_after();
            TRACE(qq ? 22 : 4, pit);
            const uint64_t v_desc = sw128_desc(smem_addr(v_smem + vs * kTileBytes), 16384, 1024);
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              // 16 keys: 2048 bytes of V, 8 TMEM columns of packed P
              mma_ts(tq + kColO, tq + kColP + 8 * kk, v_desc + 128 * kk, kIdescPV,
                     (j - 1 > j0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&sh.pv_done[qq]);
            mma_commit(&sh.v_empty[vs]);
            TRACE(qq ? 23 : 5, pit);
          }
          if (j < j1) ++it;
        }
        s = seg_end;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    // Warpgroup qq (warps 4*qq .. 4*qq+3) owns query tile qq; thread r owns row r (TMEM lane r).
    // The two warpgroups take turns for the exponentials (MUFU-bound) so that one computes
    // them while the other waits for S, loads it and reduces the row max.
    const int qq = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t t_row = tmem + kTmemPerQ * qq + ((uint32_t)((warp & 3) * 32) << 16);
    uint8_t* q_tile = q_smem + qq * kTileBytes;
    uint32_t it = 0, turns = 0;
    bool ok = true;
    // the turn barrier of this warp: its own sub-partition's, or the warpgroup's
    uint64_t* const my_turn = &sh.turn[qq][GCA_TURN_WARP ? (warp & 3) : 0];
    uint64_t* const their_turn = &sh.turn[qq ^ 1][GCA_TURN_WARP ? (warp & 3) : 0];
#if GCA_TURNS
    if (qq == 1 && (!GCA_TURN_WARP || lane == 0)) mbar_arrive(their_turn);  // query tile 0 first
#endif
    for (int64_t s = s_begin; s < s_end && ok;) {
      const int u2 = (int)(s / p.n_tiles);
      const int64_t seg_end = min(s_end, (int64_t)(u2 + 1) * p.n_tiles);
      const int j0 = (int)(s - (int64_t)u2 * p.n_tiles);
      const int j1 = (int)(seg_end - (int64_t)u2 * p.n_tiles);
      const int h = u2 / p.n_pairs;
      const int qt = (u2 % p.n_pairs) * kQPerCta + qq;
      const int qi = qt * kTileQ + r;

      // Q row -> shared memory, 128-byte swizzle (16-byte chunk c of row r at c ^ (r % 8)),
      // and its squared norm
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
      const float score_bound =
          sqrtf(q2 * __uint_as_float(p.kmax[h])) * 1.01f * p.scale_log2;

      float m_run = -INFINITY;  // running row max, log2 units (scaled)
      float l_run = 0.f;        // running row sum relative to m_run
      for (int j = j0; j < j1; ++j, ++it) {
        if (!warp_wait(&sh.s_full[qq], it & 1u, &sh, p.err)) { ok = false; break; }
        if (r == 0) TRACE(16 + qq, it);
        if (!warp_wait(&sh.lens_full[it & 3], (it >> 2) & 1u, &sh, p.err)) { ok = false; break; }
        const uint64_t lens = sh.lens[it & 3];
        if (r == 0) TRACE(6 + 5 * qq, it);
        tc_fence_after();
        float sv[kTileK];
        tmem_ld128(t_row + kColS, sv);
        tc_fence_before();
        mbar_arrive(&sh.s_free[qq]);  // the MMA warp may now compute the next S

        if (lens != 0x1010101010101010ull) {
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
        // row max: independent chains of 3-input max
        constexpr int kCh = GCA_MAX_CHAINS;
        float mx[kCh];
#pragma unroll
        for (int a = 0; a < kCh; ++a) mx[a] = fmaxf(sv[2 * a], sv[2 * a + 1]);
#pragma unroll
        for (int c = 2 * kCh; c < kTileK; c += 2 * kCh) {
#pragma unroll
          for (int a = 0; a < kCh; ++a) mx[a] = max3(mx[a], sv[c + 2 * a], sv[c + 2 * a + 1]);
        }
#pragma unroll
        for (int w = kCh / 2; w >= 1; w /= 2) {
#pragma unroll
          for (int a = 0; a < w; ++a) mx[a] = fmaxf(mx[a], mx[a + w]);
        }
        const float tile_max = mx[0] * p.scale_log2;
        if (tile_max > m_run + kRescaleThreshold) {
          m_new = tile_max;
          alpha = ex2(m_run - m_new);
        }
        }
        if (j > j0) {
          // P V of the previous tile must be done before P is overwritten or O rescaled
          if (!warp_wait(&sh.pv_done[qq], (it - 1) & 1u, &sh, p.err)) { ok = false; break; }
          tc_fence_after();
        }
        if (r == 0) TRACE(7 + 5 * qq, it);
        // P = 2^(s*c - m), inside this warpgroup's turn on MUFU: scale-subtract, exponentials,
        // bf16 packing, row sum and TMEM stores, 32 columns at a time. The turn passes to the
        // other warpgroup GCA_TURN_EARLY chunks before the end so that its first exponentials
        // queue behind this group's last ones.
#if GCA_TURNS && GCA_TURN_SPIN
        if (!__all_sync(0xffffffffu, spin_phase<(GCA_TURN_SPIN >= 2 ? GCA_TURN_SPIN : 0)>(
                                         my_turn, turns & 1u, &sh, p.err))) {
          ok = false;
          break;
        }
#elif GCA_TURNS
        if (!warp_wait(my_turn, turns & 1u, &sh, p.err)) { ok = false; break; }
#endif
        if (r == 0) TRACE(8 + 5 * qq, it);
        const float neg_m = -m_new;
#if GCA_F32X2
#pragma unroll
        for (int e = 0; e < kTileK; e += 2) fma2_pair(sv[e], sv[e + 1], p.scale_log2, neg_m);
#elif !GCA_FFMA_CHUNK
#pragma unroll
        for (int e = 0; e < kTileK; ++e) sv[e] = fmaf(sv[e], p.scale_log2, neg_m);
#endif
        float rs[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) rs[a] = 0.f;
#pragma unroll
        for (int chunk = 0; chunk < kTileK / 32; ++chunk) {
          uint32_t pk[16];
#if GCA_FFMA_CHUNK && !GCA_F32X2
#pragma unroll
          for (int e = 32 * chunk; e < 32 * chunk + 32; ++e) sv[e] = fmaf(sv[e], p.scale_log2, neg_m);
#endif
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int e = 32 * chunk + 2 * c;
            const bool poly = c < GCA_POLY_PAIRS;
            const float e0 = poly ? exp2_poly(sv[e]) : ex2(sv[e]);
            const float e1 = poly ? exp2_poly(sv[e + 1]) : ex2(sv[e + 1]);
            pk[c] = pack_bf2(e0, e1);
#if GCA_F32X2
            add2_pair(rs[2 * (c & 3)], rs[2 * (c & 3) + 1], e0, e1);
#else
            rs[2 * (c & 3)] += e0;
            rs[2 * (c & 3) + 1] += e1;
#endif
          }
          tmem_st16(t_row + kColP + 16 * chunk, reinterpret_cast<const float*>(pk));
          if (GCA_TURNS && chunk == kTileK / 32 - 1 - GCA_TURN_EARLY) {
            if (GCA_TURN_WARP) {
              __syncwarp();
              if (lane == 0) mbar_arrive(their_turn);
            } else {
              mbar_arrive(their_turn);
            }
          }
        }
        ++turns;
        if (r == 0) TRACE(9 + 5 * qq, it);
        // Lazy rescale of O (rare): after the scores are dead, before P V(j) is issued.
        if (j > j0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < kHeadDim / 16; ++c) {
            float o[16];
            tmem_ld16(t_row + kColO + 16 * c, o);
#pragma unroll
            for (int a = 0; a < 16; ++a) o[a] *= alpha;
            tmem_st16(t_row + kColO + 16 * c, o);
          }
        }
        const float row_sum =
            ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
        l_run = l_run * alpha + row_sum;
        m_run = m_new;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.p_full[qq]);
        if (r == 0) TRACE(10 + 5 * qq, it);
      }
      if (!ok) break;

      // ---- epilogue
      if (!warp_wait(&sh.pv_done[qq], (it - 1) & 1u, &sh, p.err)) break;
      tc_fence_after();
      float o[kHeadDim];
      tmem_ld64(t_row + kColO, o);
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
  }

  pdl_signal_late();
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

#if GCA_TRACE
extern "C" int gca_debug_trace(void* host, size_t bytes) {
  if (bytes > sizeof(gca::g_trace)) bytes = sizeof(gca::g_trace);
  return (int)cudaMemcpyFromSymbol(host, gca::g_trace, bytes);
}
#endif
