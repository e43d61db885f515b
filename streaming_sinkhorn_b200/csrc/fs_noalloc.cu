// fs_noalloc.cu -- fs_potentials_noalloc: the alternating solve with its scratch space taken
// from a fixed-size array in device global memory that the library owns, so the caller
// never has to allocate anything beyond its own inputs and outputs.
#include <mutex>

#include "../../include/fs.h"

namespace fs {
// Defined in fs_api.cu: the body of fs_potentials, which takes its scratch space as an
// argument; graphs_allowed = false keeps it to plain launches (instantiating a CUDA graph
// may allocate device memory, which this entry point promises not to do).
fs_status potentials_impl(const fs_problem* p, int32_t n_iters, const float* g_init, float* f,
                          float* g, void* ws, size_t ws_bytes, fs_stream_t stream,
                          bool graphs_allowed);
}

namespace {

// The scratch space. Every device that loads the library holds these bytes until the
// process exits; every call on a device reuses them.
static __device__ __align__(256) unsigned char fs_noalloc_scratch[FS_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
// The array's name in host code is only a stand-in handle, so the address must come from
// cudaGetSymbolAddress with that device current.
fs_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FS_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, fs_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return FS_ERR_CUDA;
    }
    g_scratch[dev] = ptr;
  }
  *out = g_scratch[dev];
  return FS_OK;
}

}  // namespace

extern "C" fs_status fs_potentials_noalloc(const fs_problem* p, int32_t n_iters,
                                           const float* g_init, float* f, float* g,
                                           fs_stream_t stream) {
  if (!p) return FS_ERR_NULL;
  const size_t need = fs_workspace_bytes(p);
  if (need == 0) return p->d > FS_MAX_D ? FS_ERR_UNSUPPORTED_D : FS_ERR_SHAPE;
  if (need > FS_NOALLOC_SCRATCH_BYTES) return FS_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fs_status s = scratch_address(&scratch);
  if (s != FS_OK) return s;
  // The solve clears the part of the scratch that must start at zero (its float64
  // accumulators and error word) and writes every other byte it reads, so what an
  // earlier call left there does not matter.
  return fs::potentials_impl(p, n_iters, g_init, f, g, scratch, FS_NOALLOC_SCRATCH_BYTES, stream,
                             false);
}
