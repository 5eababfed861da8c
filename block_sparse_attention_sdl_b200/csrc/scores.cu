// Block scores for anchor steps (Step-dLLM abstract: the mask is refreshed
// at anchor steps; the block-importance estimate is mean pooling of Q and K
// per block, the pooled product scaled by 1/sqrt(d), and a row softmax).
//
// Two kernels:
//   pool_kernel   reads Q and K once (16-byte streaming loads, coalesced along
//                 the contiguous (h, d) plane of each token; a warp per block
//                 and 256-element chunk) and writes fp32 block means Qbar
//                 [B,H,nb,d] and Kbar [B,H_kv,nb,d].  HBM-bound.
//   score_kernel  per (b, h, 16 query blocks): the pooled products against all
//                 Kbar rows of the KV head on the tensor cores (tf32 split in
//                 three for fp32-like accuracy), then the row softmax in shared
//                 memory.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "internal.cuh"
#include "scores_impl.cuh"

namespace sdl {
namespace {

using namespace scimpl;

template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolTensor tq, PoolTensor tk, int B,
                                                            int L, int d, int bs) {
  pool_body<T, 32, true>(tq, tk, B, L, d, bs, blockIdx.x, gridDim.x);
}

// grid: (ceil(nb / kTI), H, B); dynamic shared memory score_smem_bytes(nb, d);
// 512 threads: one 8-key tile of the pooled products and one softmax row per warp
constexpr int kScoreKernelThreads = 512;
template <int D>
__global__ void __launch_bounds__(kScoreKernelThreads, 2)
    score_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                 float* __restrict__ scores, int H, int Hkv, int nb, float scale) {
  extern __shared__ __align__(16) float sm[];
  score_body_d<D, kScoreKernelThreads>(qbar, kbar, scores, H, Hkv, nb, scale, blockIdx.x,
                                       blockIdx.y, blockIdx.z, sm);
}

}  // namespace

cudaError_t launch_pool(const void* q, const void* k, const sdl_shape& s, float* qbar,
                        float* kbar, cudaStream_t st) {
  const int nb = s.L / s.block;
  const int V = s.dtype == SDL_BF16 ? 8 : 4;
  const int per_warp = 32 * V;  // elements of the (h, d) plane per work item
  PoolTensor tq{q, qbar, s.H, (s.H * s.d + per_warp - 1) / per_warp, s.q_strides[0],
                s.q_strides[1], s.q_strides[2]};
  PoolTensor tk{k, kbar, s.H_kv, (s.H_kv * s.d + per_warp - 1) / per_warp, s.k_strides[0],
                s.k_strides[1], s.k_strides[2]};
  const int64_t items = (int64_t)s.B * nb * (tq.chunks + tk.chunks);
  const int64_t warps_per_cta = kPoolThreads / 32;
  int64_t grid = (items + warps_per_cta - 1) / warps_per_cta;
  if (grid > 148 * 16) grid = 148 * 16;  // beyond that, warps loop over items
  if (s.dtype == SDL_BF16)
    pool_kernel<__nv_bfloat16><<<(unsigned)grid, kPoolThreads, 0, st>>>(tq, tk, s.B, s.L, s.d,
                                                                        s.block);
  else
    pool_kernel<float><<<(unsigned)grid, kPoolThreads, 0, st>>>(tq, tk, s.B, s.L, s.d, s.block);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_scores_d(const float* qbar, const float* kbar, const sdl_shape& s, float scale,
                            float* scores, size_t smem, cudaStream_t st) {
  static std::atomic<bool> carveout_set[64];
  static std::atomic<size_t> smem_set[64];  // dynamic shared memory allowed so far, per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  e = once_per_device(carveout_set, [] {
    return cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared);
  });
  if (e != cudaSuccess) return e;
  // the dynamic size grows with nb; raise the kernel's allowance when needed
  if (smem > smem_set[dev].load()) {
    e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    smem_set[dev].store(smem);
  }
  const int nb = s.L / s.block;
  dim3 grid((nb + kTI - 1) / kTI, s.H, s.B);
  score_kernel<D><<<grid, kScoreKernelThreads, smem, st>>>(qbar, kbar, scores, s.H, s.H_kv, nb,
                                                           scale);
  return cudaGetLastError();
}

cudaError_t launch_scores(const float* qbar, const float* kbar, const sdl_shape& s, float scale,
                          float* scores, cudaStream_t st) {
  const size_t smem = score_smem_bytes(s.L / s.block, s.d);
  return s.d == 128 ? launch_scores_d<128>(qbar, kbar, s, scale, scores, smem, st)
                    : launch_scores_d<64>(qbar, kbar, s, scale, scores, smem, st);
}

}  // namespace sdl
