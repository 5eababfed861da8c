// Device code of the block scores (pooling, pooled products, row softmax),
// shared by the kernels of scores.cu and the fused anchor kernel of anchor.cu.
// See scores.cu for the method.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"

namespace sdl {
namespace scimpl {
namespace {  // internal linkage in every translation unit that includes this


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
__device__ __forceinline__ void pool_body(PoolTensor tq, PoolTensor tk, int B, int L, int d,
                                          int bs, int64_t bx, int64_t nbx) {
  constexpr int V = Vec<T>::N;
  const int nb = L / bs;
  const int64_t items_q = (int64_t)B * nb * tq.chunks;
  const int64_t items = items_q + (int64_t)B * nb * tk.chunks;
  const int lane = threadIdx.x % 32;
  const int64_t wpb = blockDim.x / 32;  // warps per block
  for (int64_t it = bx * wpb + threadIdx.x / 32; it < items; it += nbx * wpb) {
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

constexpr int kTI = 16;   // query blocks per CTA (4 per warp)
constexpr int kTJ = 128;  // key blocks per shared-memory tile (4 per lane)
constexpr int kScoreThreads = 128;

inline size_t score_smem_bytes(int nb, int d) {
  return sizeof(float) * ((size_t)(kTI + kTJ) * (d + 4) + (size_t)kTI * nb);
}

// Block (query-block tile bx, head h, batch element b): the first
// kScoreThreads threads do the work, any further ones of the block only join
// its barriers; shared memory `sm` of score_smem_bytes(nb, d):
//   qs [kTI][d+4], ks [kTJ][d+4], z [kTI][nb] floats.
__device__ __forceinline__ void score_body(const float* __restrict__ qbar,
                                           const float* __restrict__ kbar,
                                           float* __restrict__ scores, int H, int Hkv, int nb,
                                           int d, float scale, int bx, int h, int b, float* sm) {
  const int dp = d + 4;
  float* qs = sm;
  float* ks = qs + kTI * dp;
  float* z = ks + kTJ * dp;
  const int i0 = bx * kTI;
  const int kh = h / (H / Hkv);
  const float* qsrc = qbar + (((int64_t)b * H + h) * nb) * d;
  const float* ksrc = kbar + (((int64_t)b * Hkv + kh) * nb) * d;
  const int tid = threadIdx.x;
  const bool act = tid < kScoreThreads;
  const int d4 = d / 4;
#pragma unroll 4
  for (int x = act ? tid : kTI * d4; x < kTI * d4; x += kScoreThreads) {
    int r = x / d4, c = (x % d4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 + r < nb) v = *reinterpret_cast<const float4*>(qsrc + (int64_t)(i0 + r) * d + c);
    *reinterpret_cast<float4*>(qs + r * dp + c) = v;
  }
  const int ty = tid / 32, tx = tid % 32;
  for (int j0 = 0; j0 < nb; j0 += kTJ) {
    __syncthreads();
#pragma unroll 4
    for (int x = act ? tid : kTJ * d4; x < kTJ * d4; x += kScoreThreads) {
      int r = x / d4, c = (x % d4) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + r < nb) v = *reinterpret_cast<const float4*>(ksrc + (int64_t)(j0 + r) * d + c);
      *reinterpret_cast<float4*>(ks + r * dp + c) = v;
    }
    __syncthreads();
    if (!act) continue;
    // 4 query blocks (ty * 4 + a) x 4 key blocks (tx + 32 u) per thread: the
    // four float4 reads of keys take the 32 banks once per wavefront, the
    // query reads are broadcasts
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[a][u] = 0.f;
    for (int c = 0; c < d; c += 4) {
      float4 kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        kv[u] = *reinterpret_cast<const float4*>(ks + (tx + 32 * u) * dp + c);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float4 qv = *reinterpret_cast<const float4*>(qs + (ty * 4 + a) * dp + c);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          acc[a][u] += qv.x * kv[u].x + qv.y * kv[u].y + qv.z * kv[u].z + qv.w * kv[u].w;
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int j = j0 + tx + 32 * u;
        if (j < nb) z[(ty * 4 + a) * nb + j] = acc[a][u] * scale;
      }
    }
  }
  __syncthreads();
  // row softmax: one warp per row
  const int warp = tid / 32, lane = tid % 32;
  for (int r = act ? warp : kTI; r < kTI; r += kScoreThreads / 32) {
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
  __syncthreads();  // z may be reused by the block's next item
}

}  // namespace
}  // namespace scimpl
}  // namespace sdl
