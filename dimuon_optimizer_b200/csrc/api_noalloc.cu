// dm_step_noalloc: the optimizer step for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: a host framework whose
// caching allocator has reserved the whole device (a foreign cudaMalloc then
// fails or fragments its pool), or a latency-critical path where cudaMalloc /
// cudaFree would synchronise the device.  For them the scratch memory of the
// step lives in one file-scope device array of fixed size, created when the
// library's device code is loaded and held by every GPU that loads it until
// the process exits.  The caller still passes all inputs and outputs.
//
// The array is shared by every call: it keeps whatever the last call left in
// it.  The step zeroes the one region that must start at zero (its status
// word) and fully writes every other region before reading it.  Calls whose
// device work overlaps (two streams, two host threads without ordering)
// race on the array and must not be issued.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "dimuon.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DM_NOALLOC_MAX_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
struct ScratchSlot {
  CUcontext ctx;  // context the address belongs to
  void* ptr;
};
ScratchSlot g_scratch[MAX_DEVICES] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current driver context (null if it has none).
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// Device address of the array on the current device.  It is looked up once
// per device with that device current, and again whenever the device's
// context has changed since (after cudaDeviceReset the array belongs to a new
// module load, at a new address).  The host-side symbol itself is only a
// stand-in and must never reach a kernel.
dm_status_t scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return DM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.ptr || slot.ctx != current_context()) {
    void* p = nullptr;
    // (the look-up makes the device's primary context current if no
    // context was, so the context is read after it)
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DM_ERR_CUDA;
    slot.ptr = p;
    slot.ctx = current_context();
  }
  *out = slot.ptr;
  return DM_OK;
}

}  // namespace

extern "C" dm_status_t dm_step_noalloc(const dm_matrix_t* mats, int n, const dm_hparams_t* hp,
                                       int conditioned, int32_t* device_status_out,
                                       void* stream) {
  // Size check first: host-only, before any device call.
  size_t need = 0;
  const dm_status_t st = dm_workspace_size(mats, n, hp, conditioned, &need);
  if (st != DM_OK) return st;
  if (need > (size_t)DM_NOALLOC_MAX_BYTES) return DM_ERR_WORKSPACE;
  void* scratch = nullptr;
  const dm_status_t s2 = scratch_for_current_device(&scratch);
  if (s2 != DM_OK) return s2;
  const dm_status_t s3 =
      conditioned ? dm_dimuon_step(mats, n, hp, scratch, DM_NOALLOC_MAX_BYTES, stream)
                  : dm_muon_step(mats, n, hp, scratch, DM_NOALLOC_MAX_BYTES, stream);
  if (s3 != DM_OK) return s3;
  if (device_status_out &&
      cudaMemcpyAsync(device_status_out, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DM_ERR_CUDA;
  return DM_OK;
}
