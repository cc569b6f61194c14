// noalloc.cu -- lora_apply for callers that cannot allocate device memory.
//
// lora_apply needs a workspace for the batch plan.  Some callers cannot hand
// one over: their device memory belongs to an allocator they must not bypass
// (a framework's caching allocator, a serving runtime that pre-sizes every
// buffer), or they run in a loop that may not take the implicit device
// synchronisation cudaMalloc and cudaFree can cause.  lora_apply_noalloc
// keeps the plan in a fixed array compiled into this library instead (batches
// of at most kFusedMaxT rows need no plan: the delta kernel groups them itself
// and the array is not touched).  Every GPU that loads the library holds that
// array until the process exits.
#include <cuda.h>

#include <mutex>

#include "internal.cuh"

namespace lora {
namespace {

// Plan bytes for LORA_NOALLOC_MAX_TOKENS rows (the largest plan any accepted
// call needs; each call checks its own size).
constexpr size_t kNoAllocBytes = plan_layout(LORA_NOALLOC_MAX_TOKENS).total;

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's current context (nullptr if it cannot be read).
CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      (void)cudaGetLastError();
      return static_cast<CtxGetCurrentFn>(nullptr);
    }
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  CUcontext ctx = nullptr;
  if (fn && fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  return ctx;
}

// Device address of the scratch array on `device` (which must be current).
// The first call on a device looks it up; later calls reuse it for as long as
// the device's context is the one it was looked up in (a device reset, or a
// different driver context, makes it look up again).
int scratch_address(int device, void **out) {
  if (device < 0 || device >= kMaxDevices) return LORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  const CUcontext ctx = current_context();
  if (!g_scratch_addr[device] || ctx == nullptr || ctx != g_scratch_ctx[device]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      (void)cudaGetLastError();
      return LORA_ERR_CUDA;
    }
    g_scratch_addr[device] = ptr;
    g_scratch_ctx[device] = ctx;
  }
  *out = g_scratch_addr[device];
  return LORA_OK;
}

}  // namespace
}  // namespace lora

using namespace lora;

extern "C" int lora_apply_noalloc(lora_pool *p, int target, const void *x, int ldx, void *y, int ldy,
                                  const int32_t *ids, const float *scales, int T, void *stream) {
  NvtxRange nvtx_range("lora_apply_noalloc");
  if (!p || target < 0 || target >= p->n_targets || T < 0) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;
  if (T > LORA_NOALLOC_MAX_TOKENS || plan_layout(T).total > kNoAllocBytes) return LORA_ERR_WORKSPACE;
  if (!x || !y || !ids || !scales) return LORA_ERR_INVALID_ARG;
  const int d_in = p->targets[target].d_in, d_out = p->targets[target].d_out;
  if (ldx < d_in || ldy < d_out) return LORA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || (ldx % 8) || (ldy % 8)) return LORA_ERR_ALIGNMENT;
  const char *xa = static_cast<const char *>(x), *ya = static_cast<const char *>(y);
  if (xa < ya + size_t(T) * ldy * 2 && ya < xa + size_t(T) * ldx * 2) return LORA_ERR_INVALID_ARG;

  DeviceGuard g(p->device);
  void *ws = nullptr;
  int rc = scratch_address(p->device, &ws);
  if (rc != LORA_OK) return rc;
  // Nothing in the array needs clearing before a call: the plan kernel
  // rewrites every plan word the delta kernel reads.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DecodeCall c;
  c.targets = &target;
  c.x = x;
  c.ldx = ldx;
  c.y = y;
  c.ldy = ldy;
  c.scales = scales;
  c.T = T;
  c.ws = ws;
  if (T <= kFusedMaxT) {  // one launch, as lora_apply: the delta kernel groups the rows itself
    c.ids = ids;
    return launch_decode(p, c, st);
  }
  rc = launch_plan_ids(p, ids, T, ws, st);
  if (rc != LORA_OK) return rc;
  return launch_decode(p, c, st);
}
