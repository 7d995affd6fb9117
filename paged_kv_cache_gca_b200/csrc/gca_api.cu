// Host side of the GCA C ABI (include/gca.h): config validation, workspace layout, the host
// mirror of page counts, tensor-map setup and kernel launches. Device state lives entirely in
// the caller's workspace; the host handle holds only counters that evolve deterministically,
// so no call needs to read anything back from the GPU (only gca_check does).
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "gca_internal.h"

namespace gca {

bool nvtx_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("GCA_NVTX");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}
void nvtx_push(const char* name) { nvtxRangePushA(name); }
void nvtx_pop() { nvtxRangePop(); }

namespace {

constexpr int kMinStepsPerCta = 4;  // small launches (decode-like caches) spread wider
// Planning cost of a CTA's move to another work unit, in key-tile steps (cta_begin): measured
// per-CTA timelines put the move (epilogue, next Q tile, next first S) at ~4 us against ~1.1 us
// per step. Applied while CTAs hold 16-128 steps on average: below, ranges are too short to
// shift; above, the move is a small share of a CTA's time and the even split measured as fast.
constexpr int kUnitGapSteps = 4;
constexpr int kGapMinStepsPerCta = 16;
constexpr int kGapMaxStepsPerCta = 128;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  });
  return fn;
}

// 2D view of a page pool: rows of 64 bf16 (128 B), one row per (page, head, slot); boxes of
// 16 rows = one page of one head (2 KB), 128-byte swizzle.
bool encode_pool_map(CUtensorMap* map, void* base, int64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {(cuuint32_t)kHeadDim, (cuuint32_t)kPageSize};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

gca_status validate(const gca_config* c) {
  if (!c) return GCA_ERR_INVALID_ARG;
  if (c->num_heads < 1 || c->head_dim < 1 || c->page_size < 1 || c->grid_h < 0 ||
      c->grid_w < 0 || c->num_special < 0 || c->anchor_frames < 0 || c->window_frames < 1 ||
      c->keep_tokens < 0 || c->max_frames < 1 || c->num_pages < 1 ||
      !(c->rope_base > 0.f) || !std::isfinite(c->rope_base)) {
    return GCA_ERR_INVALID_ARG;
  }
  const int64_t P = (int64_t)c->grid_h * c->grid_w;
  const int64_t T = c->num_special + P;
  // T >= 1; a patch-free frame (grid 0 x 0) holds only its special tokens, e.g. the single
  // camera token of the causal camera head's cache
  if (T < 1 || T > (1 << 24) || c->max_frames > (1 << 24)) return GCA_ERR_INVALID_ARG;
  if (c->keep_tokens > T) return GCA_ERR_INVALID_ARG;
  if (c->keep_tokens > c->num_special && c->keep_tokens - c->num_special > P) {
    return GCA_ERR_INVALID_ARG;
  }
  if (c->head_dim != kHeadDim || c->page_size != kPageSize || c->num_heads > kMaxHeads ||
      c->keep_tokens > kMaxKeep) {
    return GCA_ERR_UNSUPPORTED;
  }
  // page rows are addressed with 32-bit coordinates
  if ((int64_t)c->num_pages * c->num_heads * kPageSize >= ((int64_t)1 << 31)) {
    return GCA_ERR_UNSUPPORTED;
  }
  return GCA_OK;
}

}  // namespace

void kept_token_list(const gca_config& c, int32_t* out, int32_t* count) {
  const int K = c.keep_tokens, S = c.num_special, P = c.grid_h * c.grid_w;
  int n = 0;
  if (K > 0) {
    if (K <= S) {
      for (int i = 0; i < K; ++i) out[n++] = i;
    } else {
      for (int i = 0; i < S; ++i) out[n++] = i;
      const int stride = P / (K - S);
      for (int j = 0; j < K - S; ++j) out[n++] = S + j * stride;
    }
  }
  *count = n;
}

bool compute_layout(const gca_config& c, Layout* L) {
  std::memset(L, 0, sizeof(*L));
  const int64_t T = c.num_special + (int64_t)c.grid_h * c.grid_w;
  const int64_t ppf = (T + kPageSize - 1) / kPageSize;
  L->T = (int32_t)T;
  L->ppf = (int32_t)ppf;
  L->last_len = (int32_t)(T - (ppf - 1) * kPageSize);
  L->n_qt = (int32_t)((T + kTileQ - 1) / kTileQ);
  const int d_sp = 2 * (c.head_dim / 6);
  L->nt = (c.head_dim - 2 * d_sp) / 2;
  L->ny = d_sp / 2;
  L->nx = d_sp / 2;
  const int64_t evicted = std::max<int64_t>(0, (int64_t)c.max_frames - c.anchor_frames -
                                                   c.window_frames);
  const int64_t traj_tokens = evicted * c.keep_tokens;
  L->traj_cap_pages = (traj_tokens + kPageSize - 1) / kPageSize + 1;
  // partial records: a launch needs 2 * (grid + units2) <= kMaxGrid + H * n_qt; the largest
  // query set is the joint prefill of the A scale frames (A * T rows)
  const int64_t max_q_rows = std::max<int64_t>(T, (int64_t)c.anchor_frames * T);
  L->part_slots = kMaxGrid + c.num_heads * (int32_t)((max_q_rows + kTileQ - 1) / kTileQ);
  const size_t page_bytes = (size_t)c.num_heads * kPageSize * c.head_dim * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = align_up(off, kAlign);
    size_t r = off;
    off += bytes;
    return r;
  };
  L->k_pool = take((size_t)c.num_pages * page_bytes);
  L->v_pool = take((size_t)c.num_pages * page_bytes);
  L->free_ring = take(4 * (size_t)c.num_pages);
  L->init_free = take(4 * (size_t)c.num_pages);
  L->seen = take(4 * (size_t)c.num_pages);
  L->frame_pages = take(4 * (size_t)c.max_frames * ppf);
  L->traj_pages = take(4 * (size_t)L->traj_cap_pages);
  L->slot_map = take(4 * (size_t)T);
  L->kept = take(4 * (size_t)kMaxKeep);
  L->rope_t = take(8 * (size_t)c.max_frames * L->nt);
  L->rope_tok = take(8 * (size_t)T * (L->ny + L->nx));
  L->err = take(4);
  L->kmax = take(4 * (size_t)c.num_heads);
  L->counters = take(8 * 4);
  L->part_o = take(4 * (size_t)L->part_slots * kTileQ * kHeadDim);
  L->part_ml = take(8 * (size_t)L->part_slots * kTileQ);
  L->total = align_up(off, kAlign);
  return true;
}

bool plan_attention(const gca_cache* c, int64_t t, int64_t max_slots, AttnParams* p,
                    bool* split, int64_t* visible_keys, int64_t q_rows) {
  const Layout& L = c->lay;
  const gca_config& cf = c->cfg;
  int64_t na_frames, w0, nwf;
  if (t < cf.anchor_frames) {
    na_frames = t + 1;
    w0 = 0;
    nwf = 0;
  } else {
    // A pending transient frame was appended without evicting: the window still holds the
    // frame that a kept append would have evicted.
    na_frames = cf.anchor_frames;
    w0 = std::max<int64_t>(cf.anchor_frames, t - cf.window_frames + (c->transient ? 0 : 1));
    nwf = t - w0 + 1;
  }
  std::memset(p, 0, sizeof(*p));
  p->frame_pages = reinterpret_cast<const int32_t*>(c->ws + L.frame_pages);
  p->traj_pages = reinterpret_cast<const int32_t*>(c->ws + L.traj_pages);
  p->err = reinterpret_cast<uint32_t*>(c->ws + L.err);
  p->kmax = reinterpret_cast<const uint32_t*>(c->ws + L.kmax);
  p->counters = reinterpret_cast<unsigned long long*>(c->ws + L.counters);
  if (q_rows <= 0) q_rows = L.T;
  const int32_t n_qt = (int32_t)((q_rows + kTileQ - 1) / kTileQ);
  p->T = (int32_t)q_rows;
  p->H = cf.num_heads;
  p->ppf = L.ppf;
  p->last_len = L.last_len;
  p->num_pages = cf.num_pages;
  p->na_pages = (int32_t)(na_frames * L.ppf);
  p->win_base = (int32_t)(w0 * L.ppf);
  p->nw_pages = (int32_t)(nwf * L.ppf);
  p->n_traj_pages = c->traj_pages;
  p->traj_tail_len =
      c->traj_pages > 0 ? (int32_t)(c->traj_len - (int64_t)(c->traj_pages - 1) * kPageSize) : 0;
  p->n_lp = p->na_pages + p->nw_pages + p->n_traj_pages;
  p->n_tiles = (p->n_lp + kPagesPerTile - 1) / kPagesPerTile;
  p->n_qt = n_qt;
  p->units = cf.num_heads * n_qt;
  p->n_pairs = (n_qt + kQPerCta - 1) / kQPerCta;
  p->units2 = cf.num_heads * p->n_pairs;
  p->total = (int64_t)p->units2 * p->n_tiles;
  int64_t gmax = std::min<int64_t>(kMaxGrid, (int64_t)c->sms * c->ctas_per_sm);
  gmax = std::min<int64_t>(gmax, max_slots / 2 - p->units2);  // partial slots must fit
  if (gmax < 1) return false;
  int64_t g = (p->total + kMinStepsPerCta - 1) / kMinStepsPerCta;
  g = std::max<int64_t>(g, std::min<int64_t>(p->units2, gmax));
  g = std::min<int64_t>(g, gmax);
  g = std::min<int64_t>(g, p->total);
  p->grid = (int32_t)g;
  p->unit_gap = (p->total >= (int64_t)kGapMinStepsPerCta * g &&
                 p->total <= (int64_t)kGapMaxStepsPerCta * g)
                    ? kUnitGapSteps
                    : 0;
  p->scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)cf.head_dim));
  p->wait_ns = c->wait_ns > 0 ? c->wait_ns : kDefaultWaitNs;
  p->withhold = c->withhold_next;
  bool sp = false;
  for (int u = 0; u < p->units2 && !sp; ++u) {
    const int64_t first = (int64_t)u * p->n_tiles;
    sp = cta_of_step(first, *p) != cta_of_step(first + p->n_tiles - 1, *p);
  }
  *split = sp;
  *visible_keys = (na_frames + nwf) * L.T + c->traj_len;
  return true;
}

// A query set of at most kDecodeMaxRows rows: one CUDA-core decode launch, the key pages of
// each head split over a cluster of dsplit CTAs (enough CTAs to cover the SMs, at least
// kDecodePagesPerSplit pages each, at most kDecodeMaxSplit).
gca_status enqueue_decode(gca_cache* c, int64_t t, int64_t visible_keys, AttnParams* p,
                          cudaStream_t s) {
  constexpr int kDecodePagesPerSplit = 8;
  const int64_t H = c->cfg.num_heads;
  int64_t S = (2 * (int64_t)c->sms + H - 1) / H;
  S = std::min<int64_t>(S, (p->n_lp + kDecodePagesPerSplit - 1) / kDecodePagesPerSplit);
  S = std::min<int64_t>(S, kDecodeMaxSplit);
  S = std::max<int64_t>(S, 1);
  p->k_pool = reinterpret_cast<const uint4*>(c->ws + c->lay.k_pool);
  p->v_pool = reinterpret_cast<const uint4*>(c->ws + c->lay.v_pool);
  p->dsplit = (int32_t)S;
  if (launch_decode(*p, s) != cudaSuccess) return GCA_ERR_CUDA;
  c->withhold_next = 0;  // the test hook applies to the tensor-core kernel only
  if (c->split_event && cudaEventRecord(c->split_event, s) != cudaSuccess) return GCA_ERR_CUDA;
  gca_attend_info& inf = c->last;
  inf.frame_idx = t;
  inf.visible_keys = visible_keys;
  inf.logical_pages = p->n_lp;
  inf.kv_tiles = p->n_tiles;
  inf.query_tiles = p->n_qt;
  inf.grid = (int32_t)(S * H);
  inf.split = S > 1 ? 1 : 0;
  inf.launches = 1;
  return GCA_OK;
}

}  // namespace gca

using namespace gca;

namespace {

template <typename T>
T* at(gca_cache* c, size_t off) {
  return reinterpret_cast<T*>(c->ws + off);
}

// Device tensors are read and written as 16-byte vectors; a misaligned pointer is rejected on
// the host instead of faulting on the device.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a + bytes) and [b, b + bytes) overlap: an attention output over its own queries would
// race (CTAs still load a unit's Q rows while others write output rows).
bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bytes && y < x + bytes;
}

bool on_cache_device(const gca_cache* c) {
  int d = -1;
  return cudaGetDevice(&d) == cudaSuccess && d == c->device;
}

}  // namespace

extern "C" {

const char* gca_status_string(gca_status s) {
  switch (s) {
    case GCA_OK: return "GCA_OK";
    case GCA_ERR_INVALID_ARG: return "GCA_ERR_INVALID_ARG";
    case GCA_ERR_OUT_OF_PAGES: return "GCA_ERR_OUT_OF_PAGES";
    case GCA_ERR_FRAME_ORDER: return "GCA_ERR_FRAME_ORDER";
    case GCA_ERR_CUDA: return "GCA_ERR_CUDA";
    case GCA_ERR_UNSUPPORTED: return "GCA_ERR_UNSUPPORTED";
    case GCA_ERR_DEVICE: return "GCA_ERR_DEVICE";
  }
  return "GCA_ERR_UNKNOWN";
}

gca_status gca_validate_config(const gca_config* cfg) { return validate(cfg); }

size_t gca_workspace_bytes(const gca_config* cfg) {
  if (validate(cfg) != GCA_OK) return 0;
  Layout L;
  compute_layout(*cfg, &L);
  return L.total;
}

gca_status gca_cache_create(const gca_config* cfg, void* dev_workspace, size_t ws_bytes,
                            const int32_t* dev_initial_free_list, void* stream,
                            gca_cache** out) {
  NvtxRange range_("gca_cache_create");
  if (!out) return GCA_ERR_INVALID_ARG;
  *out = nullptr;
  gca_status st = validate(cfg);
  if (st != GCA_OK) return st;
  Layout L;
  compute_layout(*cfg, &L);
  if (!dev_workspace || (reinterpret_cast<uintptr_t>(dev_workspace) % kAlign) != 0 ||
      ws_bytes < L.total) {
    return GCA_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(dev_initial_free_list) & 3u) != 0) return GCA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GCA_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    return GCA_ERR_CUDA;
  }
  int cc_major = 0, cc_minor = 0;
  cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (cc_major != 10 || cc_minor != 0) return GCA_ERR_UNSUPPORTED;  // built for sm_100a only

  gca_cache* c = new (std::nothrow) gca_cache;
  if (!c) return GCA_ERR_INVALID_ARG;
  std::memset(c, 0, sizeof(*c));
  c->cfg = *cfg;
  c->lay = L;
  c->ws = static_cast<char*>(dev_workspace);
  c->device = dev;
  c->sms = sms;
  kept_token_list(*cfg, c->kept, &c->n_kept);

  const int64_t rows = (int64_t)cfg->num_pages * cfg->num_heads * kPageSize;
  if (!encode_pool_map(&c->tm_k, c->ws + L.k_pool, rows) ||
      !encode_pool_map(&c->tm_v, c->ws + L.v_pool, rows)) {
    delete c;
    return GCA_ERR_CUDA;
  }
  if (attn_prepare(&c->ctas_per_sm) != cudaSuccess) {
    delete c;
    return GCA_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t page_bytes = (size_t)cfg->num_heads * kPageSize * cfg->head_dim * 2;
  bool ok = cudaMemsetAsync(c->ws + L.k_pool, 0, (size_t)cfg->num_pages * page_bytes, s) ==
                cudaSuccess &&
            cudaMemsetAsync(c->ws + L.v_pool, 0, (size_t)cfg->num_pages * page_bytes, s) ==
                cudaSuccess &&
            cudaMemsetAsync(c->ws + L.seen, 0, 4 * (size_t)cfg->num_pages, s) == cudaSuccess &&
            cudaMemsetAsync(c->ws + L.err, 0, 4, s) == cudaSuccess &&
            cudaMemsetAsync(c->ws + L.kmax, 0, 4 * (size_t)cfg->num_heads, s) == cudaSuccess &&
            cudaMemsetAsync(c->ws + L.counters, 0, 8 * 4, s) == cudaSuccess;
  if (ok) {
    InitParams ip;
    std::memset(&ip, 0, sizeof(ip));
    ip.free_ring = at<int32_t>(c, L.free_ring);
    ip.init_free = at<int32_t>(c, L.init_free);
    ip.seen = at<int32_t>(c, L.seen);
    ip.user_free = dev_initial_free_list;
    ip.kept = at<int32_t>(c, L.kept);
    ip.rope_t = at<float2>(c, L.rope_t);
    ip.rope_tok = at<float2>(c, L.rope_tok);
    ip.err = at<uint32_t>(c, L.err);
    ip.num_pages = cfg->num_pages;
    ip.max_frames = cfg->max_frames;
    ip.grid_h = cfg->grid_h;
    ip.grid_w = cfg->grid_w;
    ip.num_special = cfg->num_special;
    ip.T = L.T;
    ip.nt = L.nt;
    ip.ny = L.ny;
    ip.nx = L.nx;
    ip.keep = c->n_kept;
    ip.base = (double)cfg->rope_base;
    for (int i = 0; i < c->n_kept; ++i) ip.kept_host[i] = c->kept[i];
    ok = launch_init(ip, s) == cudaSuccess &&
         launch_check_perm(ip.seen, ip.err, cfg->num_pages, s) == cudaSuccess;
  }
  if (!ok) {
    delete c;
    return GCA_ERR_CUDA;
  }
  c->free_tail = cfg->num_pages;
  c->wait_ns = kDefaultWaitNs;
  *out = c;
  return GCA_OK;
}

namespace {

// Checks one append and fills its launch parameters from the host mirror; changes nothing.
gca_status prepare_append(gca_cache* c, int64_t t, int64_t rope_frame, uint32_t flags,
                          const void* q, const void* k, const void* v, void* q_rot_out,
                          AppendParams* out) {
  if (!c || !q || !k || !v || !q_rot_out) return GCA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_rot_out)) {
    return GCA_ERR_INVALID_ARG;
  }
  {
    // Each thread reads its own chunk of q, k, v and writes the same chunk of q_rot, so q_rot
    // may be q itself; any other overlap with q, k or v would let a thread overwrite a chunk
    // another thread has yet to read.
    const size_t bytes = (size_t)c->lay.T * c->cfg.num_heads * kHeadDim * 2;
    if ((q_rot_out != q && overlaps(q_rot_out, q, bytes)) || overlaps(q_rot_out, k, bytes) ||
        overlaps(q_rot_out, v, bytes)) {
      return GCA_ERR_INVALID_ARG;
    }
  }
  if ((flags & ~(uint32_t)GCA_APPEND_TRANSIENT) != 0u) return GCA_ERR_INVALID_ARG;
  if (t != c->frames || c->transient) return GCA_ERR_FRAME_ORDER;
  if (t >= c->cfg.max_frames) return GCA_ERR_INVALID_ARG;
  if (rope_frame < 0 || rope_frame >= c->cfg.max_frames) return GCA_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return GCA_ERR_INVALID_ARG;
  const Layout& L = c->lay;
  const gca_config& cf = c->cfg;
  const bool transient = (flags & GCA_APPEND_TRANSIENT) != 0u;
  const int64_t e = t - cf.window_frames;
  const bool evict = !transient && e >= cf.anchor_frames;
  const int K = evict ? c->n_kept : 0;
  const int64_t pages_before = (c->traj_len + kPageSize - 1) / kPageSize;
  const int64_t pages_after = (c->traj_len + K + kPageSize - 1) / kPageSize;
  const int n_pop_traj = (int)(pages_after - pages_before);
  const int64_t free_count = c->free_tail - c->free_head;
  if (L.ppf + n_pop_traj > free_count) return GCA_ERR_OUT_OF_PAGES;

  AppendParams& p = *out;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const uint4*>(q);
  p.k = static_cast<const uint4*>(k);
  p.v = static_cast<const uint4*>(v);
  p.q_rot = static_cast<uint4*>(q_rot_out);
  p.k_pool = at<uint4>(c, L.k_pool);
  p.v_pool = at<uint4>(c, L.v_pool);
  p.free_ring = at<int32_t>(c, L.free_ring);
  p.frame_pages = at<int32_t>(c, L.frame_pages);
  p.traj_pages = at<int32_t>(c, L.traj_pages);
  p.slot_map = at<int32_t>(c, L.slot_map);
  p.kept = at<int32_t>(c, L.kept);
  p.rope_t = at<float2>(c, L.rope_t);
  p.rope_tok = at<float2>(c, L.rope_tok);
  p.err = at<uint32_t>(c, L.err);
  p.kmax = at<uint32_t>(c, L.kmax);
  p.t = t;
  p.rope_frame = rope_frame;
  p.traj_len = c->traj_len;
  p.head_pos = (int32_t)(c->free_head % cf.num_pages);
  p.tail_pos = (int32_t)(c->free_tail % cf.num_pages);
  p.T = L.T;
  p.H = cf.num_heads;
  p.ppf = L.ppf;
  p.num_pages = cf.num_pages;
  p.nt = L.nt;
  p.nyx = L.ny + L.nx;
  p.evict_frame = evict ? (int32_t)e : -1;
  p.K = K;
  p.traj_pages_before = c->traj_pages;
  p.n_pop_traj = n_pop_traj;
  const int64_t end_pos = c->traj_len + K;
  p.zero_slots = (n_pop_traj > 0 && end_pos % kPageSize != 0)
                     ? (int32_t)(kPageSize - end_pos % kPageSize)
                     : 0;
  const int64_t per_tok = (int64_t)cf.num_heads * 8;
  p.tok_per_block = std::max<int32_t>(1, 256 / (int32_t)per_tok);
  p.n_tok_blocks = (int32_t)((L.ppf * kPageSize + p.tok_per_block - 1) / p.tok_per_block);
  p.n_evict_items = (int64_t)K * per_tok;
  p.n_zero_items = (int64_t)p.zero_slots * per_tok;
  p.n_push_items = evict ? L.ppf : 0;
  p.n_traj_items = n_pop_traj;
  p.n_aux_items = p.n_evict_items + p.n_zero_items + p.n_push_items + p.n_traj_items;
  const int64_t block_threads = per_tok * p.tok_per_block;
  p.n_blocks = p.n_tok_blocks + (int32_t)((p.n_aux_items + block_threads - 1) / block_threads);
  return GCA_OK;
}

// Advances the host mirror past an enqueued append.
void commit_append(gca_cache* c, const AppendParams& p, bool transient) {
  c->free_head += c->lay.ppf + p.n_pop_traj;
  if (p.evict_frame >= 0) c->free_tail += c->lay.ppf;
  c->traj_len += p.K;
  c->traj_pages += p.n_pop_traj;
  c->frames += 1;
  c->transient = transient;
}

}  // namespace

gca_status gca_append_frame_ex(gca_cache* c, int64_t t, int64_t rope_frame, uint32_t flags,
                               const void* q, const void* k, const void* v, void* q_rot_out,
                               void* stream) {
  NvtxRange range_("gca_append_frame_ex");
  AppendParams p;
  const gca_status st = prepare_append(c, t, rope_frame, flags, q, k, v, q_rot_out, &p);
  if (st != GCA_OK) return st;
  if (launch_append(p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return GCA_ERR_CUDA;
  commit_append(c, p, (flags & GCA_APPEND_TRANSIENT) != 0u);
  return GCA_OK;
}

gca_status gca_append_frame(gca_cache* c, int64_t t, const void* q, const void* k,
                            const void* v, void* q_rot_out, void* stream) {
  return gca_append_frame_ex(c, t, t, 0u, q, k, v, q_rot_out, stream);
}

gca_status gca_rollback_last_frame(gca_cache* c, int64_t t, void* /*stream*/) {
  NvtxRange range_("gca_rollback_last_frame");
  if (!c) return GCA_ERR_INVALID_ARG;
  if (!c->transient || c->frames == 0 || t != c->frames - 1) return GCA_ERR_FRAME_ORDER;
  // A transient append popped exactly ppf pages from the head and pushed none; moving the
  // head back returns them in reverse order (the ring still holds their ids).
  c->free_head -= c->lay.ppf;
  c->frames -= 1;
  c->transient = false;
  return GCA_OK;
}

gca_status gca_append_frames(gca_cache* const* caches, int32_t n, const int64_t* frame_idx,
                             const void* const* q, const void* const* k, const void* const* v,
                             void* const* q_rot_out, void* stream) {
  NvtxRange range_("gca_append_frames");
  if (!caches || !frame_idx || !q || !k || !v || !q_rot_out) return GCA_ERR_INVALID_ARG;
  if (n < 1 || n > kMaxAppendBatch) return GCA_ERR_INVALID_ARG;
  static thread_local AppendBatch b;  // ~30 KB: kept off the stack
  b.n = n;
  b.max_blocks = 0;
  for (int32_t i = 0; i < n; ++i) {
    gca_cache* c = caches[i];
    if (!c) return GCA_ERR_INVALID_ARG;
    for (int32_t j = 0; j < i; ++j) {
      if (caches[j] == c) return GCA_ERR_INVALID_ARG;  // one frame per cache per launch
    }
    if (c->device != caches[0]->device || c->lay.T != caches[0]->lay.T ||
        c->cfg.num_heads != caches[0]->cfg.num_heads) {
      return GCA_ERR_INVALID_ARG;
    }
    const gca_status st =
        prepare_append(c, frame_idx[i], frame_idx[i], 0u, q[i], k[i], v[i], q_rot_out[i], &b.p[i]);
    if (st != GCA_OK) return st;
    b.max_blocks = std::max(b.max_blocks, b.p[i].n_blocks);
  }
  if (launch_append_batch(b, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    return GCA_ERR_CUDA;
  }
  for (int32_t i = 0; i < n; ++i) commit_append(caches[i], b.p[i], false);
  return GCA_OK;
}

namespace {

// Plans and enqueues one attention of q_rows query rows (0: one frame) over the keys frame t
// sees.
gca_status enqueue_attention(gca_cache* c, int64_t t, int64_t q_rows, const void* q_rot,
                             void* out, void* stream) {
  const Layout& L = c->lay;
  AttnParams p;
  bool split = false;
  int64_t nk = 0;
  if (!plan_attention(c, t, L.part_slots, &p, &split, &nk, q_rows)) return GCA_ERR_UNSUPPORTED;
  p.q = static_cast<const uint4*>(q_rot);
  p.out = static_cast<uint4*>(out);
  p.part_o = at<float>(c, L.part_o);
  p.part_ml = at<float2>(c, L.part_ml);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p.T <= kDecodeMaxRows) return enqueue_decode(c, t, nk, &p, s);
  if (launch_attn(c->tm_k, c->tm_v, p, s) != cudaSuccess) return GCA_ERR_CUDA;
  c->withhold_next = 0;
  if (c->split_event && cudaEventRecord(c->split_event, s) != cudaSuccess) return GCA_ERR_CUDA;
  if (split && launch_combine(p, s) != cudaSuccess) return GCA_ERR_CUDA;

  gca_attend_info& inf = c->last;
  inf.frame_idx = t;
  inf.visible_keys = nk;
  inf.logical_pages = p.n_lp;
  inf.kv_tiles = p.n_tiles;
  inf.query_tiles = p.n_qt;
  inf.grid = p.grid;
  inf.split = split ? 1 : 0;
  inf.launches = split ? 2 : 1;
  return GCA_OK;
}

}  // namespace

gca_status gca_attend(gca_cache* c, int64_t t, const void* q_rot, void* out, void* stream) {
  NvtxRange range_("gca_attend");
  if (!c || !q_rot || !out || !aligned16(q_rot) || !aligned16(out)) return GCA_ERR_INVALID_ARG;
  if (c->frames == 0 || t != c->frames - 1) return GCA_ERR_FRAME_ORDER;
  if (!on_cache_device(c)) return GCA_ERR_INVALID_ARG;
  const size_t bytes = (size_t)c->lay.T * c->cfg.num_heads * kHeadDim * 2;
  if (overlaps(q_rot, out, bytes)) return GCA_ERR_INVALID_ARG;
  return enqueue_attention(c, t, 0, q_rot, out, stream);
}

gca_status gca_attend_prefill(gca_cache* c, int32_t n, const void* q_rot, void* out,
                              void* stream) {
  NvtxRange range_("gca_attend_prefill");
  if (!c || !q_rot || !out || !aligned16(q_rot) || !aligned16(out)) return GCA_ERR_INVALID_ARG;
  if (n < 1 || n > c->cfg.anchor_frames) return GCA_ERR_INVALID_ARG;
  if (c->frames != n || c->transient) return GCA_ERR_FRAME_ORDER;
  if (!on_cache_device(c)) return GCA_ERR_INVALID_ARG;
  const size_t bytes = (size_t)n * c->lay.T * c->cfg.num_heads * kHeadDim * 2;
  if (overlaps(q_rot, out, bytes)) return GCA_ERR_INVALID_ARG;
  // frames 0..n-1 are all anchors (n <= A), so frame n-1's key set is every token of them
  return enqueue_attention(c, n - 1, (int64_t)n * c->lay.T, q_rot, out, stream);
}

gca_status gca_reset(gca_cache* c, void* stream) {
  NvtxRange range_("gca_reset");
  if (!c) return GCA_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return GCA_ERR_INVALID_ARG;
  const Layout& L = c->lay;
  if (launch_reset(at<int32_t>(c, L.free_ring), at<int32_t>(c, L.init_free),
                   at<uint32_t>(c, L.err), c->cfg.num_pages,
                   static_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemsetAsync(c->ws + L.kmax, 0, 4 * (size_t)c->cfg.num_heads,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemsetAsync(c->ws + L.counters, 0, 8 * 4, static_cast<cudaStream_t>(stream)) !=
          cudaSuccess) {
    return GCA_ERR_CUDA;
  }
  c->frames = 0;
  c->free_head = 0;
  c->free_tail = c->cfg.num_pages;
  c->traj_len = 0;
  c->traj_pages = 0;
  c->transient = false;
  c->dev_err = 0;
  std::memset(&c->last, 0, sizeof(c->last));
  return GCA_OK;
}

gca_status gca_cache_destroy(gca_cache* c) {
  delete c;
  return GCA_OK;
}

gca_status gca_check(gca_cache* c) {
  NvtxRange range_("gca_check");
  if (!c) return GCA_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return GCA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return GCA_ERR_CUDA;
  uint32_t e = 0;
  if (cudaMemcpy(&e, c->ws + c->lay.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    return GCA_ERR_CUDA;
  }
  c->dev_err = e;
  return e ? GCA_ERR_DEVICE : GCA_OK;
}

gca_status gca_get_state(const gca_cache* c, gca_state* s) {
  if (!c || !s) return GCA_ERR_INVALID_ARG;
  std::memset(s, 0, sizeof(*s));
  const Layout& L = c->lay;
  s->frames_appended = c->frames;
  s->free_head = c->free_head;
  s->free_tail = c->free_tail;
  s->traj_len = c->traj_len;
  s->traj_pages = c->traj_pages;
  s->tokens_per_frame = L.T;
  s->pages_per_frame = L.ppf;
  s->pages_in_use = (int32_t)(c->cfg.num_pages - (c->free_tail - c->free_head));
  s->device_error = c->dev_err;
  s->transient = c->transient ? 1 : 0;
  s->k_pool = c->ws + L.k_pool;
  s->v_pool = c->ws + L.v_pool;
  s->free_ring = reinterpret_cast<int32_t*>(c->ws + L.free_ring);
  s->frame_pages = reinterpret_cast<int32_t*>(c->ws + L.frame_pages);
  s->traj_page_list = reinterpret_cast<int32_t*>(c->ws + L.traj_pages);
  s->slot_map = reinterpret_cast<int32_t*>(c->ws + L.slot_map);
  s->kept_tokens = reinterpret_cast<int32_t*>(c->ws + L.kept);
  return GCA_OK;
}

gca_status gca_read_attend_counters(gca_cache* c, gca_attend_counters* out) {
  NvtxRange range_("gca_read_attend_counters");
  if (!c || !out) return GCA_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return GCA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return GCA_ERR_CUDA;
  uint64_t v[4] = {0, 0, 0, 0};
  if (cudaMemcpy(v, c->ws + c->lay.counters, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
    return GCA_ERR_CUDA;
  }
  std::memset(out, 0, sizeof(*out));
  out->exact_max_rows = v[0];
  out->rescaled_rows = v[1];
  out->wide_merge_rows = v[2];
  return GCA_OK;
}

gca_status gca_set_split_event(gca_cache* c, void* cuda_event) {
  if (!c) return GCA_ERR_INVALID_ARG;
  c->split_event = static_cast<cudaEvent_t>(cuda_event);
  return GCA_OK;
}

gca_status gca_set_wait_limit(gca_cache* c, uint64_t wait_ns) {
  if (!c) return GCA_ERR_INVALID_ARG;
  c->wait_ns = wait_ns > 0 ? wait_ns : kDefaultWaitNs;
  return GCA_OK;
}

gca_status gca_test_withhold_copies(gca_cache* c) {
  if (!c) return GCA_ERR_INVALID_ARG;
  c->withhold_next = 1;
  return GCA_OK;
}

gca_status gca_last_attend_info(const gca_cache* c, gca_attend_info* info) {
  if (!c || !info) return GCA_ERR_INVALID_ARG;
  *info = c->last;
  return GCA_OK;
}

}  // extern "C"
