// fp32 block-sparse / dense attention on CUDA cores (FFMA).  Serves fp32
// inputs, whose tolerance (1e-4 absolute) the 10-bit-mantissa tensor-core
// fp32 mode cannot meet.  One CTA per 64-row query tile; two threads per
// query row, each holding half of the head dimension; key/value sub-blocks
// of 64 tokens staged in shared memory; exact online softmax per sub-block.
#include <math.h>

#include "internal.cuh"

namespace sdl {
namespace {

constexpr int kRows = 64;
constexpr int kThreads = 2 * kRows;
constexpr int kMaxSub = 1024;  // 64-token sub-blocks per sequence (L <= 65536)

template <int D>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a) {
  constexpr int DH = D / 2;
  extern __shared__ float sm[];
  float* ks = sm;                 // [64][D]
  float* vs = ks + kSubBlock * D; // [64][D]
  __shared__ uint16_t ent[kMaxSub];
  __shared__ uint32_t bits[kMaxSub / 32];
  __shared__ int n_ent;

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = tile * kRows;
  const int kh = h / (a.H / a.Hkv);
  const int nsub = a.Lk / kSubBlock;
  const int tid = threadIdx.x;

  // ---- kept 64-token key sub-blocks of this tile's query block, ascending
  for (int w = tid; w < kMaxSub / 32; w += kThreads) bits[w] = 0;
  __syncthreads();
  if (a.row_ptr == nullptr) {
    for (int s = tid; s < nsub; s += kThreads) atomicOr(&bits[s / 32], 1u << (s % 32));
  } else {
    const int i = t0 / a.block;
    const int64_t r = ((int64_t)b * a.H + h) * a.nb + i;
    const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
    const int per = a.block / kSubBlock;
    for (int x = beg + tid; x < end; x += kThreads) {
      const int j = a.col_idx[x];
      if (j < 0 || j >= a.nb || (x > beg && a.col_idx[x - 1] >= j)) {
        report_bad_mask(a.status, kBadSimtEntry, j);
        if (j < 0 || j >= a.nb) continue;
      }
      for (int u = 0; u < per; ++u) {
        const int s = j * per + u;
        atomicOr(&bits[s / 32], 1u << (s % 32));
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    const uint32_t wv = bits[tid];
    int c = __popc(wv), incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += v;
    }
    int pos = incl - c;
    for (uint32_t m = wv; m; m &= m - 1) ent[pos++] = (uint16_t)(tid * 32 + __ffs(m) - 1);
    if (tid == 31) n_ent = incl;
  }
  __syncthreads();

  // ---- this thread's query row and half of the head dimension
  const int row = tid / 2, half = tid % 2;
  const int t = t0 + row;
  const bool valid = t < a.L;
  const float* qp = reinterpret_cast<const float*>(a.q) + b * a.qs[0] + (int64_t)t * a.qs[1] +
                    h * a.qs[2] + half * DH;
  float qv[DH], acc[DH];
#pragma unroll
  for (int c = 0; c < DH; ++c) {
    qv[c] = valid ? qp[c] : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const float* kbase = reinterpret_cast<const float*>(a.k) + b * a.ks[0] + kh * a.ks[2];
  const float* vbase = reinterpret_cast<const float*>(a.v) + b * a.vs[0] + kh * a.vs[2];

  for (int e = 0; e < n_ent; ++e) {
    const int s = ent[e];
    __syncthreads();
    for (int x = tid; x < kSubBlock * D / 4; x += kThreads) {
      const int u = x / (D / 4), c = (x % (D / 4)) * 4;
      const int64_t tok = (int64_t)s * kSubBlock + u;
      *reinterpret_cast<float4*>(ks + u * D + c) =
          *reinterpret_cast<const float4*>(kbase + tok * a.ks[1] + c);
      *reinterpret_cast<float4*>(vs + u * D + c) =
          *reinterpret_cast<const float4*>(vbase + tok * a.vs[1] + c);
    }
    __syncthreads();
    float sc[kSubBlock];
    float mt = -INFINITY;
#pragma unroll 4
    for (int u = 0; u < kSubBlock; ++u) {
      const float* kr = ks + u * D + half * DH;
      float p = 0.f;
#pragma unroll
      for (int c = 0; c < DH; ++c) p = fmaf(qv[c], kr[c], p);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      sc[u] = p * a.scale;
      mt = fmaxf(mt, sc[u]);
    }
    const float mn = fmaxf(m, mt);
    const float alpha = expf(m - mn);  // m = -inf on the first sub-block -> 0
    l *= alpha;
#pragma unroll
    for (int c = 0; c < DH; ++c) acc[c] *= alpha;
    for (int u = 0; u < kSubBlock; ++u) {
      const float p = expf(sc[u] - mn);
      l += p;
      const float* vr = vs + u * D + half * DH;
#pragma unroll
      for (int c = 0; c < DH; ++c) acc[c] = fmaf(p, vr[c], acc[c]);
    }
    m = mn;
  }
  if (!valid) return;
  float* op = reinterpret_cast<float*>(a.o) + b * a.os[0] + (int64_t)t * a.os[1] + h * a.os[2] +
              half * DH;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
  for (int c = 0; c < DH; ++c) op[c] = acc[c] * inv;
  if (a.lse && half == 0) a.lse[((int64_t)b * a.H + h) * a.L + t] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t st) {
  dim3 grid((a.L + kRows - 1) / kRows, a.H, a.B);
  if (a.d == 64) {
    const size_t smem = sizeof(float) * 2 * kSubBlock * 64;
    attn_simt_kernel<64><<<grid, kThreads, smem, st>>>(a);
  } else {
    const size_t smem = sizeof(float) * 2 * kSubBlock * 128;
    cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_simt_kernel<128><<<grid, kThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sdl
