// kda_fwd_noalloc: the prefill forward for callers that cannot allocate
// device memory.
//
// kda_fwd needs a small device workspace (a status word, and for packed
// batches one int32 per sequence where the longest-first order is built).
// Some callers have no way to provide it: a hosting runtime that owns all
// device memory and forbids other allocations, or a serving loop that must
// not call cudaMalloc/cudaFree because those calls can synchronize the
// device.  This entry point takes the same inputs and outputs as kda_fwd and
// uses, instead of a caller-provided workspace, a fixed array in device
// memory that belongs to the library.  It allocates nothing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/kda.h"

namespace {

// Room for the 256-byte status word plus the order of up to
// KDA_NOALLOC_MAX_SEQUENCES packed sequences.  Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t kScratchBytes = 256 + (size_t)KDA_NOALLOC_MAX_SEQUENCES * sizeof(int32_t);
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
struct CachedAddr {
  unsigned long long ctx_id;  // driver context the address belongs to (0: none yet)
  void* addr;
};
CachedAddr g_cache[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the thread's current driver context, or 0 when there is none
// (for example right after cudaDeviceReset, before the runtime makes a new
// one).  Ids are never reused within a process, so a cached address is
// trusted only while the context that produced it is still the current one.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the array for the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// that device current and cached per device; the cache is refreshed when the
// device's context has changed since (cudaDeviceReset destroys the old one).
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = current_ctx_id();
  if (id == 0 || g_cache[dev].ctx_id != id || !g_cache[dev].addr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_cache[dev].addr = p;
    g_cache[dev].ctx_id = current_ctx_id();  // the lookup makes a context current if there was none
  }
  return g_cache[dev].addr;
}

}  // namespace

extern "C" kda_status_t kda_fwd_noalloc(const void* q, const void* k, const void* v, const float* log_alpha,
                                        const float* beta, const float* init_state, void* out,
                                        float* final_state, int B, int64_t T, int H, int dk, int dv,
                                        const int32_t* cu_seqlens, void* stream, kda_dtype_t dt) {
  if (B > KDA_NOALLOC_MAX_SEQUENCES || kda_fwd_workspace_size(B, T, H, dk, dv, dt) > kScratchBytes)
    return KDA_ERR_WORKSPACE;
  void* scratch = scratch_for_current_device();
  if (!scratch) return KDA_ERR_CUDA;
  // kda_fwd clears the status word at the start of every call and rebuilds
  // the order array, so nothing left by the previous call is read.
  return kda_fwd(q, k, v, log_alpha, beta, init_state, out, final_state, B, T, H, dk, dv, cu_seqlens, stream, dt,
                 scratch, kScratchBytes);
}

extern "C" kda_status_t kda_fwd_noalloc_status(void* stream) {
  void* scratch = scratch_for_current_device();
  if (!scratch) return KDA_ERR_CUDA;
  return kda_workspace_status(scratch, stream);
}
