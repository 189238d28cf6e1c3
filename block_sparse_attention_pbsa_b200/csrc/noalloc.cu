// pbsa_memory_update_noalloc: the persistent-memory update for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a memory-capped or
// pre-partitioned process, plug-ins whose host application owns every device
// allocation, or runtimes that forbid allocation once their pools are frozen.  They
// still own the inputs and outputs, but have no way to hand the update a workspace.
// This entry point gives them one: a fixed scratch array in the library's own device
// memory (kNoAllocScratchBytes per GPU, held from the first call until the process
// exits).  It then runs the same kernels as pbsa_memory_update.
//
// Set-up: the first call on a device looks up that device's copy of the array with
// cudaGetSymbolAddress (the array's name in host code is only a stand-in, never a
// device address) and caches the pointer; make that first call before any stream
// capture.  Every call shares the array and finds the previous call's contents in it:
// the error word is cleared on the caller's stream at the start of each call, the
// per-head completion counts of the score kernel start at zero (the array is zero when the
// library loads) and every call leaves them at zero, and the kernels write every other
// scratch byte they read.  Two calls whose work overlaps on
// the GPU (different streams, or the same stream from two threads without ordering)
// race on the array.  Device-side index errors found by this variant are recorded in
// the scratch's error word; pbsa_memory_update_noalloc_error reads and clears it (the
// next call of the update clears it too, so read it in between).
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pbsa {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB per GPU
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up once per device).
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace pbsa

extern "C" pbsa_status pbsa_memory_update_noalloc(const pbsa_geom* g, const float* q_reps, int nq,
                                                  float* k_reps, void* k_pool, void* v_pool,
                                                  int pool_slots, int* slot_gid, float* slot_ema,
                                                  int capacity, int n_sink_gid, const int* cand_slot,
                                                  const int* cand_gid, int ncand, float gamma,
                                                  int* p_list, int* p_cnt, void* stream) {
  if (nq <= 0 || capacity <= 0 || ncand < 0) return PBSA_ERR_INVALID_ARG;
  const size_t need = pbsa_workspace_bytes(g, nq, capacity + ncand);
  if (need == 0) return PBSA_ERR_INVALID_ARG;
  if (need > pbsa::kNoAllocScratchBytes) return PBSA_ERR_UNSUPPORTED;  // beyond the built-in scratch
  void* ws = nullptr;
  if (pbsa::noalloc_scratch(&ws) != cudaSuccess) return PBSA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, pbsa::WS_HEADER_BYTES, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PBSA_ERR_CUDA;
  return pbsa_memory_update(g, q_reps, nq, k_reps, k_pool, v_pool, pool_slots, slot_gid, slot_ema,
                            capacity, n_sink_gid, cand_slot, cand_gid, ncand, gamma, p_list, p_cnt,
                            ws, stream);
}

extern "C" pbsa_status pbsa_memory_update_noalloc_error(void* stream) {
  void* ws = nullptr;
  if (pbsa::noalloc_scratch(&ws) != cudaSuccess) return PBSA_ERR_CUDA;
  return pbsa_get_device_error(ws, stream);
}
