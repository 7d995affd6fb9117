// Internal declarations shared by the host API (gca_api.cu) and the kernels
// (gca_append.cu, gca_attn.cu). Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/gca.h"

struct gca_cache;

namespace gca {

constexpr int kHeadDim = 64;
constexpr int kPageSize = 16;
constexpr int kMaxHeads = 64;
constexpr int kMaxKeep = 64;
constexpr int kTileQ = 128;     // query rows per attention tile
constexpr int kTileK = 96;      // keys per attention tile (6 pages): two S/P buffers of 96
                                // columns and O (64) per query tile fill 256 TMEM columns
constexpr int kQPerCta = 2;     // query tiles per attention CTA: a work unit is a pair of tiles
                                // of one head (they share every K/V tile)
constexpr int kPagesPerTile = kTileK / kPageSize;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // bound of every attention pipeline wait
constexpr int kMaxGrid = 512;   // attention CTAs per launch (sizes the split buffers)
constexpr size_t kAlign = 1024;
constexpr int kMaxAppendBatch = 128;  // caches per batched append launch (kernel-parameter bound)

// Programmatic dependent launch: the append, attention and combine kernels are launched with
// programmatic stream serialization, signal their dependents once their main work is done and
// wait for their prerequisites (griddepcontrol.wait) before touching any data that earlier work
// in the stream produced, so a kernel's launch overlaps the previous kernel's tail. A
// prerequisite that never signals (any kernel outside this library) is waited for to its end.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches kernel<<<grid, block, smem, s>>>(args...) with programmatic stream serialization.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
#endif

// NVTX ranges around the C-ABI entry points, for timeline profilers: off unless the process
// runs with GCA_NVTX=1 (read once). With no profiler attached a range costs a function call.
bool nvtx_enabled();
void nvtx_push(const char* name);
void nvtx_pop();
struct NvtxRange {
  bool on;
  explicit NvtxRange(const char* name) : on(nvtx_enabled()) {
    if (on) nvtx_push(name);
  }
  ~NvtxRange() {
    if (on) nvtx_pop();
  }
};

// Byte offsets of every region inside the caller's workspace.
struct Layout {
  size_t k_pool, v_pool;     // bf16 [num_pages][H][16][64]
  size_t free_ring;          // int32 [num_pages]
  size_t init_free;          // int32 [num_pages] (restored by reset)
  size_t seen;               // int32 [num_pages] (permutation check at create)
  size_t frame_pages;        // int32 [max_frames][ppf]
  size_t traj_pages;         // int32 [traj_cap_pages]
  size_t slot_map;           // int32 [T]
  size_t kept;               // int32 [kMaxKeep]
  size_t rope_t;             // float2 (cos, sin) [max_frames][nt]: time band per frame
  size_t rope_tok;           // float2 (cos, sin) [T][ny + nx]: spatial bands per token
  size_t err;                // uint32 sticky device error word
  size_t kmax;               // float [H] (as uint32 bits): max squared key norm ever appended
  size_t counters;           // uint64 [4]: attention branch counters (gca_read_attend_counters)
  size_t part_o;             // float [part_slots][128][64]
  size_t part_ml;            // float2 [part_slots][128]
  size_t total;
  int64_t traj_cap_pages;
  int32_t part_slots;
  int32_t T, ppf, last_len;  // tokens per frame, pages per frame, valid slots of the last page
  int32_t n_qt;              // query tiles per head
  int32_t nt, ny, nx;        // RoPE pairs per band (t, y, x)
};

bool compute_layout(const gca_config& cfg, Layout* lay);
void kept_token_list(const gca_config& cfg, int32_t* out, int32_t* count);

// ---------------------------------------------------------------------- kernels' arguments

struct InitParams {
  int32_t* free_ring;
  int32_t* init_free;
  int32_t* seen;
  const int32_t* user_free;  // may be null
  int32_t* kept;
  float2* rope_t;
  float2* rope_tok;
  uint32_t* err;
  int32_t num_pages;
  int32_t max_frames, grid_h, grid_w, num_special, T;
  int32_t nt, ny, nx;
  int32_t keep;
  double base;
  int32_t kept_host[kMaxKeep];
};

struct AppendParams {
  const uint4* q;
  const uint4* k;
  const uint4* v;
  uint4* q_rot;
  uint4* k_pool;
  uint4* v_pool;
  int32_t* free_ring;
  int32_t* frame_pages;
  int32_t* traj_pages;
  int32_t* slot_map;
  const int32_t* kept;
  const float2* rope_t;
  const float2* rope_tok;
  uint32_t* err;
  uint32_t* kmax;  // per head: max squared key norm (float bits), raised by every append
  int64_t t;           // cache frame (page-table row)
  int64_t rope_frame;  // RoPE time position (global frame index)
  int64_t traj_len;
  int32_t head_pos;           // free_head mod num_pages: ring position of the first pop
  int32_t tail_pos;           // free_tail mod num_pages: ring position of the first push
  int32_t T, H, ppf, num_pages;
  int32_t nt, nyx;            // RoPE pairs of the time band; of the two spatial bands
  int32_t evict_frame;        // -1: nothing leaves the window
  int32_t K;                  // kept tokens copied (0 if no eviction)
  int32_t traj_pages_before;  // trajectory pages before this step
  int32_t n_pop_traj;         // trajectory pages popped by this step
  int32_t zero_slots;         // slots zero-filled at the end of the last new trajectory page
  // launch shape: token blocks of (8 chunks, H heads, tok_per_block tokens) threads, then
  // blocks of kAuxThreads for the eviction items
  int32_t tok_per_block, n_tok_blocks;
  int32_t n_blocks;  // token blocks + auxiliary blocks
  int64_t n_evict_items, n_zero_items, n_push_items, n_traj_items, n_aux_items;
};

// One frame appended to each of n caches of the same shape (T, H), in one launch: block
// (x, y) is block x of cache y's own append.
struct AppendBatch {
  int32_t n;
  int32_t max_blocks;
  AppendParams p[kMaxAppendBatch];
};
static_assert(sizeof(AppendBatch) <= 32764, "kernel parameter space");

struct AttnParams {
  const uint4* q;        // rotated queries [T][H][64] bf16
  uint4* out;            // [T][H][64] bf16
  float* part_o;         // [slots][128][64]
  float2* part_ml;       // [slots][128] (row max in log2 units, row sum)
  const int32_t* frame_pages;
  const int32_t* traj_pages;
  uint32_t* err;
  const uint32_t* kmax;  // per head: max squared key norm of everything appended
  unsigned long long* counters;  // [0] exact row max after a segment's first tile, [1] O
                                 // rescales, [2] rows merged over maxima more than 2^8 apart
  int32_t T;  // query rows of the launch (T of one frame, or n * T for a joint prefill)
  int32_t H, ppf, last_len, num_pages;
  int32_t na_pages;      // anchor pages (visible anchor frames * ppf)
  int32_t win_base;      // index into frame_pages of the first window page
  int32_t nw_pages;      // window pages
  int32_t n_traj_pages;
  int32_t traj_tail_len; // valid slots of the last trajectory page
  int32_t n_lp;          // logical pages walked
  int32_t n_tiles;       // key tiles of kTileK keys
  int32_t n_qt;          // 128-query tiles per head
  int32_t units;         // H * n_qt: (head, query tile) pairs, the combine grid
  int32_t n_pairs;       // query-tile pairs per head (a CTA works on two tiles of one head)
  int32_t units2;        // H * n_pairs: work units of the attention kernel
  int64_t total;         // units2 * n_tiles
  int32_t grid;
  int32_t unit_gap;      // planning cost of starting another work unit, in steps (cta_begin)
  float scale_log2;      // log2(e) / sqrt(D)
  uint64_t wait_ns;      // bound of every pipeline wait (a wait that runs out sets
                         // GCA_DEVERR_WAIT_TIMEOUT and the CTA winds down)
  int32_t withhold;      // test hook: 1 = CTA 0 never issues the copies of its first key tile
  // decode kernel (query sets of at most kDecodeMaxRows rows)
  const uint4* k_pool;   // [pages][H][16][64] bf16
  const uint4* v_pool;
  int32_t dsplit;        // key splits per head: one cluster of dsplit CTAs per head
};

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_init(const InitParams& p, cudaStream_t s);
cudaError_t launch_check_perm(int32_t* seen, uint32_t* err, int32_t n, cudaStream_t s);
cudaError_t launch_reset(int32_t* free_ring, const int32_t* init_free, uint32_t* err,
                         int32_t n, cudaStream_t s);
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_append_batch(const AppendBatch& b, cudaStream_t s);
cudaError_t attn_prepare(int* ctas_per_sm);  // sets kernel attributes, reports occupancy
cudaError_t launch_attn(const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                        cudaStream_t s);
cudaError_t launch_combine(const AttnParams& p, cudaStream_t s);
cudaError_t launch_decode(const AttnParams& p, cudaStream_t s);
// Enqueues the decode launch for a planned attention of at most kDecodeMaxRows query rows
// (p from plan_attention, q and out set) and records the launch in c->last.
gca_status enqueue_decode(gca_cache* c, int64_t t, int64_t visible_keys, AttnParams* p,
                          cudaStream_t s);

// Query sets of at most this many rows (the causal camera head's one camera token per frame)
// attend on CUDA cores: a 128-row tensor-core tile would be almost all padding.
constexpr int kDecodeMaxRows = 4;
constexpr int kDecodeMaxSplit = 8;  // CTAs per head: a portable cluster

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

// Split bookkeeping shared by the host planner and the attention and combine kernels. The
// flattened (pair unit, key tile) steps are cut into grid contiguous ranges of equal cost, where
// a step costs 1 and every unit is followed by unit_gap more: a CTA that moves on to another
// unit pays for that unit's start (its epilogue, the next Q tile, the next first S), so it gets
// fewer steps. In cost coordinates unit u covers [u*span, u*span + n_tiles) with span = n_tiles
// + unit_gap; CTA c starts at the step of cost c*units2*span/grid (a cut inside a gap moves to
// the next unit's start). unit_gap = 0 is the even split [c*total/grid, (c+1)*total/grid).
// (CTA c, pair unit u2, query tile q of the pair) writes its partial result to slot
// 2*(c + u2) + q; ranges are monotone, so the slots of a launch are distinct and below
// 2*(grid + units2).
__host__ __device__ inline int64_t cta_begin(int64_t c, const AttnParams& p) {
  const int64_t span = (int64_t)p.n_tiles + p.unit_gap;
  const int64_t x = c * ((int64_t)p.units2 * span) / p.grid;
  const int64_t u = x / span, off = x - u * span;
  return u * p.n_tiles + (off < p.n_tiles ? off : (int64_t)p.n_tiles);
}
// The CTA whose range holds step s (0 <= s < total): the last c with cta_begin(c) <= s. Steps
// never lie in a gap, so cta_begin(c) <= s exactly when c's cut X(c) = c*units2*span/grid is at
// most the step's cost coordinate x = u*span + (s - u*n_tiles); the last such c is
// ceil((x+1)*grid / (units2*span)) - 1 (an empty range is never returned).
__host__ __device__ inline int64_t cta_of_step(int64_t s, const AttnParams& p) {
  const int64_t span = (int64_t)p.n_tiles + p.unit_gap;
  const int64_t u = s / p.n_tiles;
  const int64_t x = u * span + (s - u * p.n_tiles);
  const int64_t tc = (int64_t)p.units2 * span;
  return ((x + 1) * p.grid + tc - 1) / tc - 1;
}
__host__ __device__ inline int64_t part_slot(int64_t cta, int64_t u2, int q) {
  return 2 * (cta + u2) + q;
}

// Fills the frame-dependent fields of p for gca_attend of frame t (visible page ranges, tiles,
// work split) with at most max_slots partial-record slots; returns false if even one CTA per
// work unit does not fit. *split: some unit spans several CTAs, so the combine kernel must run.
// q_rows: query rows of the launch (0: one frame, T).
bool plan_attention(const gca_cache* c, int64_t t, int64_t max_slots, AttnParams* p,
                    bool* split, int64_t* visible_keys, int64_t q_rows = 0);

}  // namespace gca

// Host handle of a cache (opaque in the public ABI).
struct gca_cache {
  gca_config cfg;
  gca::Layout lay;
  char* ws;
  int device;
  int sms;
  int ctas_per_sm;
  int64_t frames;
  int64_t free_head;
  int64_t free_tail;
  int64_t traj_len;
  int32_t traj_pages;
  bool transient;  // the last append was a non-keyframe awaiting rollback
  int32_t n_kept;
  int32_t kept[gca::kMaxKeep];
  uint32_t dev_err;
  uint64_t wait_ns;        // attention wait bound (gca_set_wait_limit)
  int32_t withhold_next;   // test hook armed for the next attention launch
  cudaEvent_t split_event; // measurement hook: recorded between attention and combine launches
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  gca_attend_info last;
};
