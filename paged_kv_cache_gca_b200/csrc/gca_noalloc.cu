// gca_attend_noalloc: the attention call of include/gca.h with its scratch memory taken from a
// fixed array inside this library instead of from the caller's workspace.
//
// Who needs it: some host programs may not obtain device memory after start-up at all -- for
// example a serving process that budgets every byte of the GPU when it starts and treats any
// later cudaMalloc as a failure, a plugin running inside an application whose own allocator
// owns the device, or a latency-critical loop in which a cudaMalloc (which can synchronise the
// device) is not allowed. This entry point allocates nothing, ever: its only scratch is
// g_attend_scratch below, a 16 MiB array that every GPU which loads the library holds until
// the process exits.
//
// What the scratch holds: when a frame's keys are split across CTAs, each CTA leaves a partial
// record (unnormalised O rows, row max, row sum) that the combine kernel merges. Every slot
// that is read has been written earlier in the same call, so nothing needs clearing; the array
// keeps the last call's contents. All calls of this entry point share the one array: two calls
// whose kernels overlap on the GPU (different streams, or different caches on different
// streams) race on it, so callers must order them (one stream, or events).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "gca_internal.h"

namespace gca {
namespace {

constexpr size_t kNoallocScratchBytes = (size_t)16 << 20;
constexpr size_t kSlotOBytes = (size_t)kTileQ * kHeadDim * sizeof(float);
constexpr size_t kSlotMLBytes = (size_t)kTileQ * sizeof(float2);
constexpr int kNoallocSlots = (int)(kNoallocScratchBytes / (kSlotOBytes + kSlotMLBytes));
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_attend_scratch[kNoallocScratchBytes];

// Device address of g_attend_scratch per device. In host code the symbol's name is only a
// host-side stand-in, so the address is looked up with the device current, once per device and
// CUDA context: the address is cached next to the context it was taken in and looked up again
// when the device's current context is a different one (after a cudaDeviceReset, or when the
// caller destroyed and re-created the primary context), so a stale address is never used.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
  });
  return fn;
}

struct ScratchEntry {
  CUcontext ctx;
  void* addr;
};
std::mutex g_scratch_mutex;
ScratchEntry g_scratch[kMaxDevices] = {};

cudaError_t scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (!get_ctx) return cudaErrorNotSupported;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
  if (!ctx || !g_scratch[dev].addr || g_scratch[dev].ctx != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attend_scratch);  // also makes a context
    if (e != cudaSuccess) return e;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorContextIsDestroyed;
    g_scratch[dev].ctx = ctx;
    g_scratch[dev].addr = p;
  }
  *out = g_scratch[dev].addr;
  return cudaSuccess;
}

}  // namespace
}  // namespace gca

using namespace gca;

extern "C" gca_status gca_attend_noalloc(gca_cache* c, int64_t t, const void* q_rot, void* out,
                                         void* stream) {
  NvtxRange range_("gca_attend_noalloc");
  if (!c || !q_rot || !out) return GCA_ERR_INVALID_ARG;
  // 16-byte vector accesses: a misaligned tensor is rejected here, not faulted on the device
  if (((reinterpret_cast<uintptr_t>(q_rot) | reinterpret_cast<uintptr_t>(out)) & 15u) != 0) {
    return GCA_ERR_INVALID_ARG;
  }
  if (c->frames == 0 || t != c->frames - 1) return GCA_ERR_FRAME_ORDER;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != c->device) return GCA_ERR_INVALID_ARG;
  {  // an output over its own queries would race
    const uintptr_t x = reinterpret_cast<uintptr_t>(q_rot), y = reinterpret_cast<uintptr_t>(out);
    const size_t bytes = (size_t)c->lay.T * c->cfg.num_heads * kHeadDim * 2;
    if (x < y + bytes && y < x + bytes) return GCA_ERR_INVALID_ARG;
  }
  // The partial records of one call must fit the array (at least one CTA per work unit).
  AttnParams p;
  bool split = false;
  int64_t nk = 0;
  if (!plan_attention(c, t, kNoallocSlots, &p, &split, &nk)) return GCA_ERR_UNSUPPORTED;
  if (p.T <= kDecodeMaxRows) {  // the decode kernel merges its splits on chip: no scratch
    p.q = static_cast<const uint4*>(q_rot);
    p.out = static_cast<uint4*>(out);
    return enqueue_decode(c, t, nk, &p, static_cast<cudaStream_t>(stream));
  }
  void* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return GCA_ERR_CUDA;
  p.q = static_cast<const uint4*>(q_rot);
  p.out = static_cast<uint4*>(out);
  p.part_o = static_cast<float*>(scratch);
  p.part_ml = reinterpret_cast<float2*>(static_cast<char*>(scratch) +
                                        (size_t)kNoallocSlots * kSlotOBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_attn(c->tm_k, c->tm_v, p, s) != cudaSuccess) return GCA_ERR_CUDA;
  c->withhold_next = 0;
  if (split && launch_combine(p, s) != cudaSuccess) return GCA_ERR_CUDA;
  return GCA_OK;
}
