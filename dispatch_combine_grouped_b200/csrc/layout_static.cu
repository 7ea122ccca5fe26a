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
// the device address is looked up once per device with cudaGetSymbolAddress, with that
// device current, and cached.
#include <mutex>

#include "kernels.cuh"

namespace moe {

// Enough for N*k <= 131072 assignments with E <= 256 and P <= 32 (1.65 MB needed).
constexpr size_t kNoAllocScratchBytes = 2u << 20;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_layout_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
static cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_layout_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace moe

extern "C" moe_status moe_dispatch_layout_noalloc(const moe_config* cfg, const int32_t* expert_owner,
                                                  const int32_t* topk_ids, const moe_layout* out,
                                                  int32_t* dev_status, moe_stream_t stream) {
  using namespace moe;
  moe_status s = moe_check_config(cfg);
  if (s != MOE_OK) return s;
  if (!expert_owner && cfg->E % cfg->P != 0) return MOE_ERR_INVALID_ARG;
  if (!out || !out->n_e || !out->expert_off || !out->C || !out->send_off || !out->recv_off || !out->tok2send ||
      !out->send2row || !out->ret2tok || !out->tok2row || !out->row2tok || !out->tile_off ||
      (cfg->N > 0 && !topk_ids))
    return MOE_ERR_INVALID_ARG;
  // the same scratch size moe_dispatch_layout asks for; beyond the array: refuse
  if (moe_layout_workspace_bytes(cfg) > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  // Every scratch word the layout kernels read is written earlier in the same call, so
  // the previous call's contents need no clearing.
  if (launch_layout(*cfg, expert_owner, topk_ids, *out, dev_status, scratch, (cudaStream_t)stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
