// tq_scores_noalloc: attention logits for callers that cannot allocate device
// memory.
//
// Some callers have no way to obtain a device buffer: code running under an
// allocator that forbids cudaMalloc (a fixed memory budget handed out once at
// start-up), plug-ins whose host framework owns every allocation, or glue code
// in languages with no binding for CUDA's allocator.  tq_scores needs a
// caller-supplied workspace; this variant instead uses a scratch array compiled
// into the library.
//
// The scratch is one file-scope __device__ array of TQ_SCORES_NOALLOC_SCRATCH
// bytes.  Every GPU that loads the library holds it until the process exits.
// Host code must not hand the array's name to a kernel: on the host that name
// is only a stand-in for the device object, not a device address.  The address
// is looked up with cudaGetSymbolAddress once per device, with that device
// current, the first time this entry point runs on the device, and cached.
// Make that first call before any stream capture, because the lookup may load
// the module.  The cached address belongs to the device's primary context: a
// device reset (cudaDeviceReset) destroys it, so no call of this entry point
// may follow one in the same process.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  Calls whose kernels overlap on the GPU (different streams, or several
// host threads) race on it, so callers must serialise them.  The scoring path
// writes every scratch word it reads before reading it, so nothing in the
// scratch needs clearing between calls.
#include <cuda_runtime.h>

#include <mutex>

#include "tq_internal.h"
#include "tq_trace.h"

#define TQ_SCORES_NOALLOC_SCRATCH (2u << 20)  // 2 MiB
#define TQ_NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char g_tq_scores_scratch[TQ_SCORES_NOALLOC_SCRATCH];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_addr[TQ_NOALLOC_MAX_DEVICES] = {};

// Device address of the scratch array on `device` (which must be current).
tq_status scratch_address(int device, void** out) {
  if (device < 0 || device >= TQ_NOALLOC_MAX_DEVICES)
    return tq_fail(TQ_ERR_UNSUPPORTED, "tq_scores_noalloc: device %d outside 0..%d", device,
                   TQ_NOALLOC_MAX_DEVICES - 1);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_tq_scores_scratch);
    if (e != cudaSuccess || !p)
      return tq_fail(TQ_ERR_CUDA, "tq_scores_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return TQ_OK;
}
}  // namespace

extern "C" tq_status tq_scores_noalloc(const tq_codec* kc, const void* q, tq_dtype dtype, int B, int Hq, int Hkv,
                                       int64_t T, const tq_compressed* K, float* logits, void* stream) {
  const tqtrace::Range trace("tq_scores_noalloc");
  if (!kc) return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores_noalloc: null codec");
  if (kc->device < 0) return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores_noalloc: host-only codec");
  size_t need = 0;
  tq_status st = tq_scores_workspace_size(kc, B, Hq, Hkv, &need);
  if (st != TQ_OK) return st;
  if (need > TQ_SCORES_NOALLOC_SCRATCH)
    return tq_fail(TQ_ERR_UNSUPPORTED,
                   "tq_scores_noalloc: B=%d, Hq=%d, Hkv=%d needs %zu bytes of scratch, above the built-in %u "
                   "bytes; use tq_scores with a workspace",
                   B, Hq, Hkv, need, (unsigned)TQ_SCORES_NOALLOC_SCRATCH);
  int cur = -1;
  const cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return tq_fail(TQ_ERR_CUDA, "tq_scores_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (cur != kc->device)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores_noalloc: current device %d is not the codec's device %d", cur,
                   kc->device);
  void* scratch = nullptr;
  if ((st = scratch_address(cur, &scratch)) != TQ_OK) return st;
  return tq_scores(kc, q, dtype, B, Hq, Hkv, T, K, logits, scratch, TQ_SCORES_NOALLOC_SCRATCH, stream);
}
