/*
 * gca.h -- C ABI of the B200 (sm_100a) paged KV cache for Geometric Context Attention.
 *
 * One cache serves one attention layer of a streaming video transformer. Every frame:
 *   1. its tokens' q and k get 3D (t, y, x) rotary embeddings, t being the global frame index
 *      ("How the Geometric Context Transformer Enables Streaming 3D Reconstruction in
 *      LingBot-Map", section "3D Rotary Positional Embeddings");
 *   2. its k (rotated) and v are appended to device pages; the frame that left the sliding
 *      window is evicted, keeping only a few tokens in the trajectory pool
 *      (same page, section "FlashInferBlock": append_frame, then evict_frames);
 *   3. its queries attend with an online softmax over three pools -- anchor frame(s), the window
 *      of recent frames and the trajectory pool ("LingBot-Map runs 10,000 frames on monocular
 *      video", section "How GCT's Anchor-Pose-Trajectory Pools Make Monocular 3D Tractable";
 *      FlashInferBlock: compute_attention).
 *
 * Conventions fixed by this library where the pages are silent:
 *   - token order in a frame: camera, registers, then patches row-major over (grid_h, grid_w);
 *   - RoPE: bands d_y = d_x = 2*floor(D/6), d_t = D - d_y - d_x in the order (t, y, x);
 *     interleaved pairs (2j, 2j+1); pair j of a band of width d turns by pos * base^(-2j/d);
 *     a patch at row r, column c is at (t, r+1, c+1); camera/register tokens at (t, 0, 0);
 *   - window W counts the current frame; at frame t the window is frames max(A, t-W+1)..t and
 *     frame t-W (if >= A) is evicted; anchors (frames 0..A-1) are never evicted;
 *   - kept tokens of an evicted frame: K <= S: tokens 0..K-1; otherwise all S special tokens
 *     plus patches S + j*floor(P/(K-S)), j = 0..K-S-1;
 *   - attention scale 1/sqrt(D); no mask inside the current frame; frame-causal across frames
 *     (except the joint prefill of the first scale frames, gca_attend_prefill);
 *   - pages: FIFO free list; a frame takes ceil(T/page_size) pages (page-aligned); the
 *     trajectory pool is dense (page_size tokens per page) and never freed; the evicted
 *     frame's pages go back to the tail of the free list in row order.
 *
 * Tensors are raw device pointers, bf16, contiguous, token-major "NHD": [T][H][D], 16-byte
 * aligned (the kernels move them in 16-byte vectors; a misaligned pointer is rejected with
 * GCA_ERR_INVALID_ARG). A device initial free list must be 4-byte aligned.
 * Streams are cudaStream_t passed as void* (NULL = legacy default stream).
 * Calls that enqueue work never synchronise; only gca_check() does.
 * Supported sizes: head_dim 64, page_size 16, 1 <= num_heads <= 64, keep_tokens <= 64.
 */
#ifndef GCA_H_
#define GCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gca_cache gca_cache; /* opaque host handle */

typedef enum {
  GCA_OK = 0,
  GCA_ERR_INVALID_ARG = -1,  /* bad pointer, size or config value */
  GCA_ERR_OUT_OF_PAGES = -2, /* the step needs more free pages than the pool has */
  GCA_ERR_FRAME_ORDER = -3,  /* frame_idx is not the next frame (append) / last frame (attend) */
  GCA_ERR_CUDA = -4,         /* a CUDA runtime call failed */
  GCA_ERR_UNSUPPORTED = -5,  /* valid but not implemented size (e.g. head_dim != 64) */
  GCA_ERR_DEVICE = -6        /* a kernel set the cache's sticky device error word */
} gca_status;

/* Device error bits (gca_state.device_error after gca_check). */
#define GCA_DEVERR_PAGE_RANGE 0x1u   /* a page id read from device state was out of range */
#define GCA_DEVERR_WAIT_TIMEOUT 0x2u /* a pipeline wait in the attention kernel gave up */
#define GCA_DEVERR_FREE_LIST 0x4u    /* the initial free list is not a permutation */
#define GCA_DEVERR_SMEM_ALIGN 0x8u   /* attention kernel: shared memory base not 1024-aligned */

typedef struct {
  int32_t num_heads;     /* H */
  int32_t head_dim;      /* D; 64 */
  int32_t page_size;     /* tokens per page; 16 */
  int32_t grid_h;        /* patch rows per frame (0 with no patches) */
  int32_t grid_w;        /* patch columns per frame (0 with no patches) */
  int32_t num_special;   /* S: camera + register tokens; T = S + grid_h * grid_w >= 1 (a
                          * patch-free cache, e.g. the causal camera head's: T = S = 1) */
  int32_t anchor_frames; /* A >= 0 */
  int32_t window_frames; /* W >= 1, counts the current frame */
  int32_t keep_tokens;   /* K >= 0 tokens kept per evicted frame (0: no trajectory pool) */
  int32_t max_frames;    /* cache frames one stream may hold before gca_reset, and the RoPE
                          * table length (every RoPE time position is < max_frames) */
  int32_t num_pages;     /* physical page capacity of the pool */
  float rope_base;       /* RoPE theta (> 0, finite) */
} gca_config;

/* Host-mirrored counters and device addresses of a cache's state. Filling it never touches the
 * GPU. All device arrays live inside the caller's workspace. */
typedef struct {
  int64_t frames_appended;
  int64_t free_head;    /* the free list is ring[(free_head .. free_tail-1) mod num_pages] */
  int64_t free_tail;
  int64_t traj_len;     /* tokens in the trajectory pool */
  int32_t traj_pages;   /* pages held by the trajectory pool */
  int32_t tokens_per_frame;
  int32_t pages_per_frame;
  int32_t pages_in_use;
  uint32_t device_error; /* last value read by gca_check() */
  int32_t transient;     /* 1 while the last append is a non-keyframe awaiting rollback */
  void* k_pool;          /* bf16 [num_pages][H][page_size][D]: rotated keys */
  void* v_pool;          /* bf16 [num_pages][H][page_size][D]: values */
  int32_t* free_ring;    /* int32 [num_pages] */
  int32_t* frame_pages;  /* int32 [max_frames][pages_per_frame]: page row of every frame */
  int32_t* traj_page_list; /* int32 [trajectory page capacity] */
  int32_t* slot_map;     /* int32 [T]: page*page_size + slot of the last appended frame's tokens */
  int32_t* kept_tokens;  /* int32 [K]: token indices an evicted frame keeps */
} gca_state;

/* Work description of the last gca_attend() or gca_attend_prefill() call (host values, for
 * measurement; gca_attend_noalloc does not update it). */
typedef struct {
  int64_t frame_idx;
  int64_t visible_keys;  /* Nk(t): keys the frame's queries see */
  int32_t logical_pages; /* pages walked, incl. partially filled ones */
  int32_t kv_tiles;      /* 96-key tiles per query tile */
  int32_t query_tiles;   /* 128-query tiles per head */
  int32_t grid;          /* CTAs of the attention kernel */
  int32_t split;         /* 1 if any (head, query tile) was split across CTAs (combine ran) */
  int32_t launches;      /* kernels enqueued by the call */
} gca_attend_info;

/* Counts of the attention kernels' data-dependent branches since create / the last gca_reset
 * (all attention and combine launches of the cache). A "row" is one query row of one head. */
typedef struct {
  uint64_t exact_max_rows;  /* (row, key tile) pairs past a work piece's first tile whose exact
                             * row max was computed: the bound |q| max|k| did not rule out a
                             * rescale */
  uint64_t rescaled_rows;   /* (row, key tile) pairs where the running max grew by more than
                             * 2^8 and O was rescaled in tensor memory */
  uint64_t wide_merge_rows; /* rows the split-KV combine merged from pieces whose row maxima lie
                             * more than 2^8 apart */
  uint64_t reserved;
} gca_attend_counters;

/* Validates a config. Host only. Returns GCA_OK, GCA_ERR_INVALID_ARG or GCA_ERR_UNSUPPORTED. */
gca_status gca_validate_config(const gca_config* cfg);

/* Bytes of device workspace a cache with this config needs (0 if the config is invalid).
 * Host only; the size does not depend on the GPU. */
size_t gca_workspace_bytes(const gca_config* cfg);

/* Creates a cache inside a caller-owned device workspace (>= gca_workspace_bytes, 1024-byte
 * aligned). Enqueues initialisation on `stream` (zeroed pools, RoPE tables, free list).
 * dev_initial_free_list: NULL for the order 0..num_pages-1, else a device array int32
 * [num_pages] holding a permutation (the free list's initial order; copied, and restored by
 * gca_reset). A non-permutation sets GCA_DEVERR_FREE_LIST, reported by gca_check.
 * The workspace must stay allocated until gca_cache_destroy. Ownership: the caller owns the
 * workspace; the library owns only *out. The GPU current at this call is the cache's device. */
gca_status gca_cache_create(const gca_config* cfg, void* dev_workspace, size_t ws_bytes,
                            const int32_t* dev_initial_free_list, void* stream,
                            gca_cache** out);

/* Appends frame `frame_idx` (pages' append_frame, then evict_frames):
 * RoPE on q and k, k_rot and v scattered into freshly popped pages, q_rot written for
 * gca_attend, and the frame that leaves the window evicted (kept tokens copied to the
 * trajectory tail, its pages pushed back to the free list) -- one kernel launch.
 * q, k, v: device bf16 [T][H][D]; q_rot_out: device bf16 [T][H][D]: it may be q itself, but
 * any other overlap with q, k or v is rejected (GCA_ERR_INVALID_ARG).
 * frame_idx must equal the number of frames appended since create/reset
 * (GCA_ERR_FRAME_ORDER) and be < max_frames. The page budget is checked on the host from
 * mirrored counts: GCA_ERR_OUT_OF_PAGES returns with nothing enqueued. */
gca_status gca_append_frame(gca_cache* cache, int64_t frame_idx, const void* q, const void* k,
                            const void* v, void* q_rot_out, void* stream);

/* Flags of gca_append_frame_ex. */
enum {
  /* A non-keyframe (pages' skip_append path, keyframe-only caching): the frame's K/V are
   * appended and it may be attended, but nothing is evicted, and gca_rollback_last_frame must
   * follow before the next append. While it is pending, gca_attend of this frame sees the
   * anchors, the window frames still cached plus this one (up to W+1 frames) and the
   * trajectory. */
  GCA_APPEND_TRANSIENT = 1
};

/* gca_append_frame with an explicit RoPE time position and flags. frame_idx is the cache
 * frame (the number of frames kept so far: non-keyframes do not count once rolled back);
 * rope_frame is the global index of the video frame (the time position of its 3D RoPE;
 * 0 <= rope_frame < max_frames). gca_append_frame(c, t, ...) is
 * gca_append_frame_ex(c, t, t, 0, ...). Errors as gca_append_frame, and GCA_ERR_FRAME_ORDER
 * while a transient frame awaits rollback; GCA_ERR_INVALID_ARG for unknown flags. */
gca_status gca_append_frame_ex(gca_cache* cache, int64_t frame_idx, int64_t rope_frame,
                               uint32_t flags, const void* q, const void* k, const void* v,
                               void* q_rot_out, void* stream);

/* Undoes the transient append of frame frame_idx (pages' rollback_last_frame): the frame's
 * pages return to the head of the free list in reverse order, which restores the allocator
 * exactly, and the frame count goes back to frame_idx. Host bookkeeping only: nothing is
 * enqueued (the device ring still holds the page ids at those positions; the pages' contents
 * are left as they are and are overwritten when popped again). Work already enqueued that
 * reads the frame (its gca_attend) must be ordered before the next append, which is the case
 * on one stream. GCA_ERR_FRAME_ORDER unless the last append was transient and was frame
 * frame_idx. `stream` is unused. */
gca_status gca_rollback_last_frame(gca_cache* cache, int64_t frame_idx, void* stream);

/* gca_append_frame for n caches at once, in one kernel launch: cache caches[i] appends frame
 * frame_idx[i] from q[i], k[i], v[i] and writes q_rot_out[i]. The caches are distinct, on one
 * device, with the same tokens per frame and head count (other settings, e.g. window, RoPE
 * base and page budget, may differ); 1 <= n <= 128. All arrays are host arrays of length n
 * holding device pointers (q, k, v, q_rot_out as for gca_append_frame). Each cache's result is
 * bit-identical to its own gca_append_frame call. All-or-nothing: the first failing check
 * (GCA_ERR_INVALID_ARG, GCA_ERR_FRAME_ORDER, GCA_ERR_OUT_OF_PAGES) returns with nothing
 * enqueued and no cache changed. A single 12 MB append is too short to reach HBM bandwidth;
 * batching the appends of several caches (the layers' or streams' caches of one step) in one
 * launch is how the append runs near copy bandwidth. The pages append per cache; the batched
 * form is an addition of this library. */
gca_status gca_append_frames(gca_cache* const* caches, int32_t n, const int64_t* frame_idx,
                             const void* const* q, const void* const* k, const void* const* v,
                             void* const* q_rot_out, void* stream);

/* Attention of the last appended frame's queries over the cache (pages' compute_attention):
 * out[i][h] = softmax_j(q_rot[i][h] . k_j[h] / sqrt(D)) v_j[h] over the anchor, window and
 * trajectory keys visible at frame frame_idx (which must be the last appended frame).
 * q_rot: device bf16 [T][H][D] from gca_append_frame; out: device bf16 [T][H][D], not
 * overlapping q_rot (GCA_ERR_INVALID_ARG: CTAs still read queries while others write rows).
 * One tcgen05 attention launch, plus one combine launch when the key range is split. A frame
 * of at most 4 tokens (the causal camera head's cache: one camera token per frame) attends on
 * CUDA cores instead, in one launch: per head a cluster of up to 8 CTAs splits the key pages
 * and merges in on-chip shared memory (gca_attend_info: launches 1, grid = splits * H). */
gca_status gca_attend(gca_cache* cache, int64_t frame_idx, const void* q_rot, void* out,
                      void* stream);

/* Joint attention of the first n frames (the scale frames), bidirectional: after exactly n
 * appends (n <= anchor_frames, so all n frames are anchors), the n*T queries of frames 0..n-1
 * attend over every token of those frames, with no mask across frames (pages: the scale frames
 * are processed jointly with bidirectional attention, then streaming switches to causal;
 * Streaming Inference API, FAQ on scale frames). q_rot: device bf16 [n*T][H][D], the q_rot
 * outputs of the n appends back to back (frame-major); out: device bf16 [n*T][H][D], not
 * overlapping q_rot (GCA_ERR_INVALID_ARG). One
 * attention launch (+ one combine launch when split; n*T <= 4 query rows: the one-launch CUDA-
 * core path of gca_attend). GCA_ERR_INVALID_ARG unless
 * 1 <= n <= anchor_frames; GCA_ERR_FRAME_ORDER unless exactly n frames are appended (and no
 * transient frame is pending). */
gca_status gca_attend_prefill(gca_cache* cache, int32_t n, const void* q_rot, void* out,
                              void* stream);

/* The same attention as gca_attend, for callers that may not allocate device memory while
 * they run: a process that budgets all GPU memory when it starts and treats any later
 * cudaMalloc as a failure, a plugin whose host application owns the device allocator, or a
 * latency-critical loop where a cudaMalloc (which can synchronise the device) is not allowed.
 * It allocates nothing. Its scratch -- the split-KV partial records -- lives in a 16 MiB array
 * inside this library, which every GPU that loads the library holds until the process exits.
 * The first call on a device looks up that array's device address (cudaGetSymbolAddress) with
 * the device current; under CUDA's lazy module loading that is also when the device commits the
 * array's 16 MiB. Make that first call before any stream capture; later calls allocate nothing. The address is kept with
 * the CUDA context it was taken in and looked up again when the context changes (for example
 * after a cudaDeviceReset). All calls share the one
 * array and it keeps the last call's contents (every slot read is written earlier in the same
 * call): calls whose kernels overlap on the GPU race on it, so order them (one stream, or
 * events). The array holds 496 partial records of 128 query rows; a launch over num_heads *
 * ceil(T / 256) query-tile pairs needs two per pair and two per CTA, so this returns
 * GCA_ERR_UNSUPPORTED when num_heads * ceil(T / 256) >= 248; other errors as gca_attend.
 * A frame of at most 4 tokens takes gca_attend's CUDA-core path, which needs no scratch (and
 * does not touch the array).
 * The web pages have no counterpart of this entry point; it is an addition of this library. */
gca_status gca_attend_noalloc(gca_cache* cache, int64_t frame_idx, const void* q_rot, void* out,
                              void* stream);

/* Restores the state of a new stream (pages' clean_kv_cache): free list back to its initial
 * order, counters to zero, device error word cleared. Enqueued on `stream`. */
gca_status gca_reset(gca_cache* cache, void* stream);

/* Frees the host handle. Never frees the caller's workspace. NULL is accepted. */
gca_status gca_cache_destroy(gca_cache* cache);

/* Synchronises the device, reads the sticky device error word into the state and returns
 * GCA_ERR_DEVICE if it is non-zero. Once the word is set, every later attention of the cache
 * does nothing (its output is left unwritten) until gca_reset; appends keep running, every
 * page id range-checked before any write, so the pools stay in bounds. */
gca_status gca_check(gca_cache* cache);

/* Synchronises the device and reads the cache's attention branch counters (for tests and
 * measurement: they show which paths of the online softmax a stream exercised). The decode path
 * of frames of at most 4 tokens keeps a plain online softmax and counts nothing. */
gca_status gca_read_attend_counters(gca_cache* cache, gca_attend_counters* counters);

/* Measurement hook: while cuda_event (a cudaEvent_t created by the caller) is set, every
 * gca_attend / gca_attend_prefill of this cache records it on the call's stream right after the
 * attention kernel's launch and before the combine's (after the single launch of the decode
 * path), so that events around the call split its
 * time between the two kernels. NULL clears it. An event between the launches stops the combine
 * from starting early (programmatic launch), so use it in a separate, instrumented pass. */
gca_status gca_set_split_event(gca_cache* cache, void* cuda_event);

/* Bound of every pipeline wait inside this cache's attention kernels, in nanoseconds (0 restores
 * the default, 2 s). A wait that runs out -- which only a stalled pipeline can cause -- sets
 * GCA_DEVERR_WAIT_TIMEOUT in the sticky device error word; the kernel's CTAs then stop issuing
 * work, wait (bounded) for the copies and MMAs they already issued, free their tensor memory and
 * return, so the call always ends and the CUDA context stays usable. Host only; applies to
 * attention launches enqueued after the call. The decode kernel of frames of at most 4 tokens has
 * no pipeline waits. */
gca_status gca_set_wait_limit(gca_cache* cache, uint64_t wait_ns);

/* Test hook of the timeout path above. Arms the next attention launch of this cache
 * (gca_attend, gca_attend_prefill or gca_attend_noalloc): in it, CTA 0 never issues the copies
 * of its first key tile (nothing is ever in flight for that tile), so its MMA issuer's wait for
 * them runs out after the wait limit and the launch sets GCA_DEVERR_WAIT_TIMEOUT. The combine
 * launch of the call then does nothing (sticky error), so no output row that depends on a
 * split work unit is written; gca_check reports GCA_ERR_DEVICE until gca_reset. One-shot; a call
 * that takes the decode path (at most 4 query rows) clears it without effect. */
gca_status gca_test_withhold_copies(gca_cache* cache);

/* Fills *state from the host mirror (no GPU access). */
gca_status gca_get_state(const gca_cache* cache, gca_state* state);

/* Fills *info for the last gca_attend() call (host only). */
gca_status gca_last_attend_info(const gca_cache* cache, gca_attend_info* info);

/* Human-readable name of a status. */
const char* gca_status_string(gca_status status);

#ifdef __cplusplus
}
#endif

#endif /* GCA_H_ */
