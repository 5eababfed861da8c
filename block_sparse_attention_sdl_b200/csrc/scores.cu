// Block scores for anchor steps (Step-dLLM abstract: the mask is refreshed
// at anchor steps; the block-importance estimate is mean pooling of Q and K
// per block, the pooled product scaled by 1/sqrt(d), and a row softmax).
//
// Two kernels:
//   pool_kernel   reads Q and K once (16-byte vector loads, coalesced along the
//                 contiguous (h, d) plane of each token, one warp per block and
//                 256-element chunk) and writes fp32 block means Qbar
//                 [B,H,nb,d] and Kbar [B,H_kv,nb,d].  HBM-bound.
//   score_kernel  per (b, h, 16 query blocks): fp32 FFMA products against all
//                 Kbar rows of the KV head, then the row softmax in shared memory.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "scores_impl.cuh"

namespace sdl {
namespace {

using namespace scimpl;

template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolTensor tq, PoolTensor tk, int B,
                                                            int L, int d, int bs) {
  pool_body<T>(tq, tk, B, L, d, bs, blockIdx.x, gridDim.x);
}

// grid: (ceil(nb / kTI), H, B); dynamic shared memory score_smem_bytes(nb, d)
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              float* __restrict__ scores, int H,
                                                              int Hkv, int nb, int d,
                                                              float scale) {
  extern __shared__ float sm[];
  score_body(qbar, kbar, scores, H, Hkv, nb, d, scale, blockIdx.x, blockIdx.y, blockIdx.z, sm);
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

cudaError_t launch_scores(const float* qbar, const float* kbar, const sdl_shape& s, float scale,
                          float* scores, cudaStream_t st) {
  const int nb = s.L / s.block;
  const size_t smem = score_smem_bytes(nb, s.d);
  static std::atomic<bool> attr_set[64];  // per device; the maximum size is constant
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                227 * 1024);
  });
  if (e != cudaSuccess) return e;
  dim3 grid((nb + kTI - 1) / kTI, s.H, s.B);
  score_kernel<<<grid, kScoreThreads, smem, st>>>(qbar, kbar, scores, s.H, s.H_kv, nb, s.d, scale);
  return cudaGetLastError();
}

}  // namespace sdl
