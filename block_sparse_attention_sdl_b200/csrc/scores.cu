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

namespace sdl {
namespace {

constexpr int kPoolThreads = 256;

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(float (&acc)[8], const uint4& u) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(p[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void add(float (&acc)[4], const uint4& u) {
    acc[0] += __uint_as_float(u.x);
    acc[1] += __uint_as_float(u.y);
    acc[2] += __uint_as_float(u.z);
    acc[3] += __uint_as_float(u.w);
  }
};

struct PoolTensor {
  const void* x;
  float* out;
  int Hx;
  int chunks;  // 32-lane chunks of the (h, d) plane
  int64_t s0, s1, s2;
};

// One warp per work item (tensor, b, block i, chunk of 32 lanes x 16 bytes of
// the contiguous (h, d) plane): each lane sums its elements over the block's
// tokens with independent 16-byte loads, then writes the means.  Items of Q
// come first, then those of K.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolTensor tq, PoolTensor tk, int B,
                                                            int L, int d, int bs) {
  constexpr int V = Vec<T>::N;
  const int nb = L / bs;
  const int64_t items_q = (int64_t)B * nb * tq.chunks;
  const int64_t items = items_q + (int64_t)B * nb * tk.chunks;
  const int lane = threadIdx.x % 32;
  for (int64_t it = ((int64_t)blockIdx.x * kPoolThreads + threadIdx.x) / 32; it < items;
       it += (int64_t)gridDim.x * (kPoolThreads / 32)) {
    const bool isq = it < items_q;
    const PoolTensor& tx = isq ? tq : tk;
    const int64_t r = isq ? it : it - items_q;
    const int chunk = (int)(r % tx.chunks);
    const int i = (int)((r / tx.chunks) % nb);
    const int b = (int)(r / ((int64_t)tx.chunks * nb));
    const int e = (chunk * 32 + lane) * V;  // element of the (h, d) plane
    if (e >= tx.Hx * d) continue;
    const int h = e / d, c = e % d;
    const T* base = reinterpret_cast<const T*>(tx.x) + b * tx.s0 + h * tx.s2 + c +
                    (int64_t)i * bs * tx.s1;
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
#pragma unroll 16
    for (int t = 0; t < bs; ++t) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)t * tx.s1));
      Vec<T>::add(acc, u);
    }
    const float inv = 1.0f / (float)bs;
    float* dst = tx.out + (((int64_t)b * tx.Hx + h) * nb + i) * d + c;
#pragma unroll
    for (int v = 0; v < V; v += 4)
      *reinterpret_cast<float4*>(dst + v) =
          make_float4(acc[v] * inv, acc[v + 1] * inv, acc[v + 2] * inv, acc[v + 3] * inv);
  }
}

constexpr int kTI = 16;  // query blocks per CTA (4 per warp)
constexpr int kTJ = 64;  // key blocks per shared-memory tile
constexpr int kScoreThreads = 128;

// grid: (ceil(nb / kTI), H, B).  Dynamic shared memory:
//   qs [kTI][d+4], ks [kTJ][d+4], z [kTI][nb] floats.
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              float* __restrict__ scores, int H,
                                                              int Hkv, int nb, int d,
                                                              float scale) {
  extern __shared__ float sm[];
  const int dp = d + 4;
  float* qs = sm;
  float* ks = qs + kTI * dp;
  float* z = ks + kTJ * dp;
  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * kTI;
  const int kh = h / (H / Hkv);
  const float* qsrc = qbar + (((int64_t)b * H + h) * nb) * d;
  const float* ksrc = kbar + (((int64_t)b * Hkv + kh) * nb) * d;
  const int tid = threadIdx.x;
  const int d4 = d / 4;
  for (int x = tid; x < kTI * d4; x += kScoreThreads) {
    int r = x / d4, c = (x % d4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 + r < nb) v = *reinterpret_cast<const float4*>(qsrc + (int64_t)(i0 + r) * d + c);
    *reinterpret_cast<float4*>(qs + r * dp + c) = v;
  }
  const int ty = tid / 32, tx = tid % 32;
  for (int j0 = 0; j0 < nb; j0 += kTJ) {
    __syncthreads();
    for (int x = tid; x < kTJ * d4; x += kScoreThreads) {
      int r = x / d4, c = (x % d4) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + r < nb) v = *reinterpret_cast<const float4*>(ksrc + (int64_t)(j0 + r) * d + c);
      *reinterpret_cast<float4*>(ks + r * dp + c) = v;
    }
    __syncthreads();
    float acc[4][2];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = 0.f;
    for (int c = 0; c < d; c += 4) {
      float4 kv0 = *reinterpret_cast<const float4*>(ks + tx * dp + c);
      float4 kv1 = *reinterpret_cast<const float4*>(ks + (tx + 32) * dp + c);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float4 qv = *reinterpret_cast<const float4*>(qs + (ty * 4 + a) * dp + c);
        acc[a][0] += qv.x * kv0.x + qv.y * kv0.y + qv.z * kv0.z + qv.w * kv0.w;
        acc[a][1] += qv.x * kv1.x + qv.y * kv1.y + qv.z * kv1.z + qv.w * kv1.w;
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        int j = j0 + tx + 32 * u;
        if (j < nb) z[(ty * 4 + a) * nb + j] = acc[a][u] * scale;
      }
    }
  }
  __syncthreads();
  // row softmax: one warp per row
  const int warp = tid / 32, lane = tid % 32;
  for (int r = warp; r < kTI; r += kScoreThreads / 32) {
    if (i0 + r >= nb) break;
    float* zr = z + r * nb;
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, zr[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
    for (int j = lane; j < nb; j += 32) {
      float e = expf(zr[j] - m);
      zr[j] = e;
      s += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv = 1.0f / s;
    float* dst = scores + (((int64_t)b * H + h) * nb + (i0 + r)) * nb;
    for (int j = lane; j < nb; j += 32) dst[j] = zr[j] * inv;
  }
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
  const size_t smem = sizeof(float) * ((size_t)(kTI + kTJ) * (s.d + 4) + (size_t)kTI * nb);
  static bool attr_set = false;  // the attribute is per function; max size is constant
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((nb + kTI - 1) / kTI, s.H, s.B);
  score_kernel<<<grid, kScoreThreads, smem, st>>>(qbar, kbar, scores, s.H, s.H_kv, nb, s.d, scale);
  return cudaGetLastError();
}

}  // namespace sdl
