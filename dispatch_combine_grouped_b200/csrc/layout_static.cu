// moe_dispatch_layout_noalloc: the dispatch layout for callers that cannot allocate GPU
// memory.
//
// Some callers have no way to hand this library a workspace: a plugin that runs inside
// another runtime which owns every device buffer, a serving loop that must never call
// cudaMalloc (it synchronises the whole device and can stall every other stream), or a
// service with a fixed memory budget decided at start-up.  This entry point runs the
// same three layout kernels as moe_dispatch_layout, but their scratch lives in a
// fixed-size array compiled into the library, so the caller passes only the ids and the
// layout arrays.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kNoAllocScratchBytes for it until the process exits.  Host code cannot use the
// array's name as a device address (on the host it names a host-side placeholder), so
// the device address is looked up with cudaGetSymbolAddress, with the device current,
// on the first call on each device, and cached.  The cache remembers the context it was
// looked up in: after a device reset (cudaDeviceReset, or anything else that destroys
// the primary context) the module is loaded again at another address, so the next call
// looks the address up again instead of writing through a stale one.
#include <mutex>

#include "kernels.cuh"

namespace moe {

// Enough for N*k <= 131072 assignments with E <= 256 and P <= 32 (1.65 MB needed).
constexpr size_t kNoAllocScratchBytes = 2u << 20;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_layout_scratch[kNoAllocScratchBytes];

struct NoAllocSlot {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;
};

static std::mutex g_noalloc_mu;
static NoAllocSlot g_noalloc[kNoAllocMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if the driver cannot say).
static unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device (looked up on the first
// call in each context, with the device current).
static cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc[dev];
  // no context yet (id 0), or another one than the address was looked up in: look up
  // again (cudaGetSymbolAddress also brings up the primary context if needed)
  if (slot.ptr == nullptr || slot.ctx_id == 0 || slot.ctx_id != current_context_id()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_layout_scratch);
    if (e != cudaSuccess) return e;
    slot.ptr = p;
    slot.ctx_id = current_context_id();
  }
  *out = slot.ptr;
  return cudaSuccess;
}

}  // namespace moe

extern "C" moe_status moe_dispatch_layout_noalloc(const moe_config* cfg, const int32_t* expert_owner,
                                                  const int32_t* topk_ids, const moe_layout* out,
                                                  int32_t* dev_status, moe_stream_t stream) {
  using namespace moe;
  moe_status s = moe_check_config(cfg);  // records its own message
  if (s != MOE_OK) return s;
  if (!expert_owner && cfg->E % cfg->P != 0)
    return record_error(MOE_ERR_INVALID_ARG, "contiguous placement needs E % P == 0");
  if (!out || !out->n_e || !out->expert_off || !out->C || !out->send_off || !out->recv_off || !out->tok2send ||
      !out->send2row || !out->ret2tok || !out->tok2row || !out->row2tok || !out->tile_off)
    return record_error(MOE_ERR_INVALID_ARG, "every layout array must be non-NULL");
  if (cfg->N > 0 && !topk_ids) return record_error(MOE_ERR_INVALID_ARG, "topk_ids is NULL");
  // the same scratch size moe_dispatch_layout asks for; beyond the array: refuse
  if (moe_layout_workspace_bytes(cfg) > kNoAllocScratchBytes)
    return record_error(MOE_ERR_UNSUPPORTED, "layout scratch exceeds the built-in 2 MiB array "
                                             "(moe_layout_workspace_bytes(cfg) > 2 MiB)");
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return record_cuda_error(e, "layout (noalloc): scratch address");
  // Every scratch word the layout kernels read is written earlier in the same call, so
  // the previous call's contents need no clearing.
  return record_cuda_error(launch_layout(*cfg, expert_owner, topk_ids, *out, dev_status, scratch,
                                         (cudaStream_t)stream),
                           "layout (noalloc)");
}
