// fs_noalloc.cu -- fs_potentials_noalloc: the alternating solve with its scratch space taken
// from a fixed-size array in device global memory that the library owns, so the caller
// never has to allocate anything beyond its own inputs and outputs.
#include "../../include/fs.h"

namespace fs {
// Defined in fs_api.cu: the body of fs_potentials, which takes its scratch space as an
// argument; graphs_allowed = false keeps it to plain launches (instantiating a CUDA graph
// may allocate device memory, which this entry point promises not to do).
fs_status potentials_impl(const fs_problem* p, int32_t n_iters, const float* g_init, float* f,
                          float* g, void* ws, size_t ws_bytes, fs_stream_t stream,
                          bool graphs_allowed);
// Defined in fs_api.cu: keeps the text of a CUDA error for fs_last_cuda_error.
void record_cuda_error(const char* what, cudaError_t e);
}

namespace {

// The scratch space. Every device whose context has loaded this file's module holds these
// bytes until the process exits; every call on a device reuses them.
static __device__ __align__(256) unsigned char fs_noalloc_scratch[FS_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current context. The array's name in host
// code is only a stand-in handle, so the address must come from cudaGetSymbolAddress with
// the device (and context) current that the kernels will run in. It is looked up on every
// call, never cached: after cudaDeviceReset, or under another context of the same device,
// the module is loaded anew and the array may sit at another address. Once the module is
// loaded the lookup is a host-side table query. Under lazy module loading (the default
// since CUDA 12.2) the first lookup in a context loads the module, which commits the
// array's device memory; when the device cannot provide it the call returns
// FS_ERR_DEVICE_MEMORY.
fs_status scratch_address(void** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, fs_noalloc_scratch);
  if (e != cudaSuccess || !ptr) {
    fs::record_cuda_error("cudaGetSymbolAddress(fs_noalloc_scratch)", e);
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? FS_ERR_DEVICE_MEMORY : FS_ERR_CUDA;
  }
  *out = ptr;
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
