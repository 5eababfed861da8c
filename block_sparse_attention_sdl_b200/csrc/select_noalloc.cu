// sdl_select_mask_noalloc: mask selection for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: code that runs inside a
// device-memory pool's own callbacks (where calling the allocator again would
// re-enter it), or a serving process that reserves its whole memory budget at
// start-up and forbids any cudaMalloc afterwards.  This entry point runs the
// same selection kernels as sdl_select_mask, but their scratch lives in a
// fixed array compiled into this library instead of a caller workspace.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes.
// Every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address, so the first call on
// each device looks its address up with cudaGetSymbolAddress (with that device
// current) and caches it; make that first call before any stream capture.
// No call allocates: no cudaMalloc, cudaFree or allocating library routine.
//
// All calls share the one array, and it keeps whatever the previous call left
// in it (the kernels clear what must start at zero).  Calls that can overlap
// on the GPU -- on different streams, or from different host threads --
// race on the array: serialize them.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.cuh"

namespace sdl {
namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;  // 2 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace sdl

extern "C" sdl_status sdl_select_mask_noalloc(const float* scores, const sdl_shape* shape,
                                              double sparsity, int32_t* row_ptr,
                                              int32_t* col_idx, int64_t col_capacity,
                                              uint8_t* mask_u8, void* stream) {
  const size_t need = sdl_select_workspace_bytes(shape);
  if (need == 0) return SDL_ERR_INVALID_ARG;  // bad shape
  if (!scores || !row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  const int64_t total = sdl_mask_budget(shape, sparsity);
  if (total < 0) return SDL_ERR_INVALID_ARG;
  if (col_capacity < total) return SDL_ERR_CAPACITY;
  if (need > sdl::kNoAllocScratchBytes) return SDL_ERR_WORKSPACE;  // beyond the fixed array
  void* scratch = nullptr;
  cudaError_t e = sdl::scratch_address(&scratch);
  if (e != cudaSuccess) return SDL_ERR_CUDA;
  return sdl_select_mask(scores, shape, sparsity, row_ptr, col_idx, col_capacity, mask_u8,
                         scratch, sdl::kNoAllocScratchBytes, stream);
}
