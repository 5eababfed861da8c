// Column-sparse attention of the PulseCol abstract: every query head keeps a
// set of key tokens (columns of the attention matrix) for all of its query
// rows, chosen at a refresh step and reused until the next one.
//
// The abstract gives no estimator or budget; the reading implemented here:
//   score:  S[b,h,u] = (1/nb) * sum over query blocks i of
//           softmax over u of (scale * Qbar[b,h,i,:] . k[b,u,h/g,:])
//   budget: Lc = 64 * floor((1 - s) * L / 64 + 0.5) columns per head, at
//           least 64 (whole 64-key tiles)
//   select: the Lc largest S[b,h,:] of each head, ties to the lower u,
//           listed in ascending u
//   attend: softmax over the kept keys only, for every query token of the head
//
// Kernels:
//   col_stats_kernel  per (b, h, 128 query blocks, 512 keys): row max and
//                     sum of exp of the block-mean queries' logits over those
//                     keys (fp32 FFMA, 128 x 128 tiles, 8 x 8 per thread);
//   col_combine_kernel per row: its maximum and sum over all keys, merged
//                     from the partials in key order;
//   col_sum_kernel    per (b, h, 128 keys): the column sums of the softmax
//                     weights, over the query blocks in a fixed order (no
//                     atomics: the same bits on every run).
//   col_select_kernel per (b, h): radix select of the Lc-th largest score
//                     (digits of 11, 11, 10 bits), then the kept columns in
//                     ascending order.
//   col_gather_kernel the kept K and V tokens into dense [B, Lc, H, d]
//                     tensors (one per query head); the attention kernel then
//                     walks them as dense keys (attn_tc.cu, key length Lc).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "select_impl.cuh"

namespace sdl {
namespace {

using selimpl::block_excl_scan;

struct ColArgs {
  int B, H, Hkv, L, d, nb;
  float scale;
  int64_t ks[3], vs[3];  // (b, t, h) strides of K and V, in elements
};

void fill_col_args(ColArgs& c, const sdl_shape& s, float scale) {
  c.B = s.B;
  c.H = s.H;
  c.Hkv = s.H_kv;
  c.L = s.L;
  c.d = s.d;
  c.nb = s.L / s.block;
  c.scale = scale;
  for (int i = 0; i < 3; ++i) {
    c.ks[i] = s.k_strides[i];
    c.vs[i] = s.v_strides[i];
  }
}

// Score tiles: 128 query blocks x 128 keys per CTA of 256 threads, each thread
// 8 x 8 logits (rows ty + 16 r, keys tx + 16 j), fp32 FFMA over d from shared
// memory (rows padded by 4 floats: the float4 reads of 16 keys hit every bank
// once per pair of wavefronts, the 2 rows of a warp are broadcasts).
constexpr int kGR = 128;       // query blocks per tile
constexpr int kGK = 128;       // keys per tile
constexpr int kGT = 256;       // threads
constexpr int kGKT = 4;        // key tiles per CTA of the statistics pass

inline int col_groups(int L) { return ((L + kGK - 1) / kGK + kGKT - 1) / kGKT; }
// qs [kGR][d+4] (block-mean queries), ks [kGK][d+4] (keys as fp32)
inline size_t col_smem_bytes(int d) { return sizeof(float) * (size_t)(kGR + kGK) * (d + 4); }
constexpr size_t kColSumExtra = sizeof(float) * (16 * kGK + 2 * kGR);

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// Rows i0 .. i0+kGR of Qbar (head h) into qs; zero rows past nb.
__device__ __forceinline__ void load_q_tile(const float* __restrict__ qsrc, int nb, int d, int i0,
                                            float* qs) {
  const int dp = d + 4, d4 = d / 4;
  for (int x = threadIdx.x; x < kGR * d4; x += kGT) {
    const int r = x / d4, c = (x % d4) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 + r < nb) v = *reinterpret_cast<const float4*>(qsrc + (int64_t)(i0 + r) * d + c);
    *reinterpret_cast<float4*>(qs + r * dp + c) = v;
  }
}

// Keys u0 .. u0+kGK of KV head kh into ks (fp32; zero past L), 16 bytes per
// load (the (b, t, h) strides are multiples of 16 bytes and d of 8 elements).
template <typename T>
__device__ __forceinline__ void load_k_tile(const T* __restrict__ k, const int64_t* ks, int b,
                                            int kh, int d, int u0, int L, float* kt) {
  constexpr int V = 16 / sizeof(T);  // elements per load
  const int dp = d + 4, dv = d / V;
#pragma unroll 4
  for (int x = threadIdx.x; x < kGK * dv; x += kGT) {
    const int r = x / dv, c = (x % dv) * V;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (u0 + r < L)
      u = __ldg(reinterpret_cast<const uint4*>(k + b * ks[0] + (int64_t)(u0 + r) * ks[1] +
                                               kh * ks[2] + c));
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int y = 0; y < V; y += 4)
      *reinterpret_cast<float4*>(kt + r * dp + c + y) =
          make_float4(to_f<T>(e[y]), to_f<T>(e[y + 1]), to_f<T>(e[y + 2]), to_f<T>(e[y + 3]));
  }
}

// z[r][j] = scale * (qs row ty + 16 r) . (ks row tx + 16 j), summed over d in order.
__device__ __forceinline__ void tile_logits(const float* qs, const float* kt, int d, float scale,
                                            float (&z)[8][8]) {
  const int dp = d + 4, ty = threadIdx.x / 16, tx = threadIdx.x % 16;
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int j = 0; j < 8; ++j) z[r][j] = 0.f;
#pragma unroll 1
  for (int c = 0; c < d; c += 4) {
    float4 a[8], bv[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) a[r] = *reinterpret_cast<const float4*>(qs + (ty + 16 * r) * dp + c);
#pragma unroll
    for (int j = 0; j < 8; ++j) bv[j] = *reinterpret_cast<const float4*>(kt + (tx + 16 * j) * dp + c);
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float t = fmaf(a[r].x, bv[j].x, z[r][j]);
        t = fmaf(a[r].y, bv[j].y, t);
        t = fmaf(a[r].z, bv[j].z, t);
        z[r][j] = fmaf(a[r].w, bv[j].w, t);
      }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int j = 0; j < 8; ++j) z[r][j] *= scale;
}

// Statistics pass.  grid (col_groups(L), ceil(nb / kGR), B * H): for its
// query blocks and its kGKT key tiles, part[bh, i, group] = (max over those
// keys of z_iu, sum of exp(z_iu - max)).
template <typename T>
__global__ void __launch_bounds__(kGT) col_stats_kernel(const float* __restrict__ qbar,
                                                        const T* __restrict__ k, ColArgs c,
                                                        float2* __restrict__ part) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* kt = qs + kGR * (c.d + 4);
  const int bh = blockIdx.z, b = bh / c.H, h = bh % c.H, i0 = blockIdx.y * kGR;
  const int kh = h / (c.H / c.Hkv);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const int ngroups = gridDim.x;
  load_q_tile(qbar + (int64_t)bh * c.nb * c.d, c.nb, c.d, i0, qs);
  float m[8], l[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
  }
  for (int t = 0; t < kGKT; ++t) {
    const int u0 = (blockIdx.x * kGKT + t) * kGK;
    if (u0 >= c.L) break;
    __syncthreads();
    load_k_tile<T>(k, c.ks, b, kh, c.d, u0, c.L, kt);
    __syncthreads();
    float z[8][8];
    tile_logits(qs, kt, c.d, c.scale, z);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (u0 + tx + 16 * j >= c.L)  // no such key
#pragma unroll
        for (int r = 0; r < 8; ++r) z[r][j] = -INFINITY;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float mt = m[r];
#pragma unroll
      for (int j = 0; j < 8; ++j) mt = fmaxf(mt, z[r][j]);
      float acc = l[r] * expf(m[r] - mt);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc += expf(z[r][j] - mt);
      l[r] = acc;
      m[r] = mt;
    }
  }
  // merge the 16 key lanes' partial (max, sum) of each row, in a fixed order
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    for (int o = 8; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m[r], o);
      const float l2 = __shfl_xor_sync(0xffffffffu, l[r], o);
      const float mt = fmaxf(m[r], m2);
      l[r] = (mt == -INFINITY) ? 0.f : l[r] * expf(m[r] - mt) + l2 * expf(m2 - mt);
      m[r] = mt;
    }
    const int i = i0 + ty + 16 * r;
    if (tx == 0 && i < c.nb)
      part[((int64_t)bh * c.nb + i) * ngroups + blockIdx.x] = make_float2(m[r], l[r]);
  }
}

// stats[bh, i] = (max, 1 / sum) of row i over all keys, from its groups in order.
__global__ void col_combine_kernel(const float2* __restrict__ part, int rows, int ngroups,
                                   float2* __restrict__ stats) {
  const int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= rows) return;
  const float2* p = part + x * ngroups;
  float m = -INFINITY, l = 0.f;
  for (int g = 0; g < ngroups; ++g) {
    const float2 v = p[g];
    const float mt = fmaxf(m, v.x);
    if (mt == -INFINITY) continue;
    l = l * expf(m - mt) + v.y * expf(v.x - mt);
    m = mt;
  }
  stats[x] = make_float2(m, 1.0f / l);
}

// Sum pass.  grid (ceil(L / kGK), B * H): S[bh, u] = (1/nb) sum over i of
// exp(z_iu - max_i) / sum_i, the query blocks in order (no atomics: the same
// bits on every run).
template <typename T>
__global__ void __launch_bounds__(kGT) col_sum_kernel(const float* __restrict__ qbar,
                                                      const T* __restrict__ k, ColArgs c,
                                                      const float2* __restrict__ stats,
                                                      float* __restrict__ S) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* kt = qs + kGR * (c.d + 4);
  float* red = kt + kGK * (c.d + 4);  // [16][kGK]: per row group ty, per key
  float* rm = red + 16 * kGK;         // [kGR] row maxima of the tile
  float* rinv = rm + kGR;             // [kGR] inverse row sums
  const int bh = blockIdx.y, b = bh / c.H, h = bh % c.H, u0 = blockIdx.x * kGK;
  const int kh = h / (c.H / c.Hkv);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  load_k_tile<T>(k, c.ks, b, kh, c.d, u0, c.L, kt);
  const float* qsrc = qbar + (int64_t)bh * c.nb * c.d;
  const float2* st = stats + (int64_t)bh * c.nb;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int i0 = 0; i0 < c.nb; i0 += kGR) {
    __syncthreads();
    load_q_tile(qsrc, c.nb, c.d, i0, qs);
    for (int x = threadIdx.x; x < kGR; x += kGT) {
      const float2 v = i0 + x < c.nb ? st[i0 + x] : make_float2(0.f, 0.f);
      rm[x] = v.x;
      rinv[x] = v.y;
    }
    __syncthreads();
    float z[8][8];
    tile_logits(qs, kt, c.d, c.scale, z);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int ri = ty + 16 * r;
      if (i0 + ri < c.nb) {
        const float mr = rm[ri], ir = rinv[ri];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += expf(z[r][j] - mr) * ir;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[ty * kGK + tx + 16 * j] = acc[j];
  __syncthreads();
  for (int x = threadIdx.x; x < kGK && u0 + x < c.L; x += kGT) {
    float t = 0.f;
    for (int w = 0; w < 16; ++w) t += red[w * kGK + x];
    S[(int64_t)bh * c.L + u0 + x] = t / (float)c.nb;
  }
}

constexpr int kSelThreads = 1024;

// grid B * H: cols[bh, 0 .. Lc) = the Lc largest S[bh, :] (ties: lower u), ascending.
__global__ void __launch_bounds__(kSelThreads) col_select_kernel(const float* __restrict__ S,
                                                                 int L, int Lc,
                                                                 int32_t* __restrict__ cols) {
  __shared__ int hist[2048];
  __shared__ int s_warp[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_krem;
  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.x;
  const uint32_t* keys = reinterpret_cast<const uint32_t*>(S + bh * L);  // scores >= 0
  int32_t* out = cols + bh * Lc;
  uint32_t prefix = 0;
  int krem = Lc;  // the Lc-th largest key
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const int width = p < 2 ? 11 : 10, shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
    const int nbin = 1 << width, hs = shift + width;
    for (int x = tid; x < nbin; x += kSelThreads) hist[x] = 0;
    __syncthreads();
    for (int u = tid; u < L; u += kSelThreads) {
      const uint32_t key = keys[u];
      if (hs >= 32 || (key >> hs) == (prefix >> hs))
        atomicAdd(&hist[(key >> shift) & (uint32_t)(nbin - 1)], 1);
    }
    __syncthreads();
    // thread t owns bins [nbin - per (t+1), nbin - per t): the top bins first
    const int per = nbin / kSelThreads;  // 2 or 1
    const int hi = nbin - per * tid;
    int cnt[2] = {0, 0}, local = 0;
    for (int x = 0; x < per; ++x) {
      cnt[x] = hist[hi - 1 - x];
      local += cnt[x];
    }
    int total = 0;
    int above = block_excl_scan(local, s_warp, total);
    for (int x = 0; x < per; ++x) {
      if (above < krem && above + cnt[x] >= krem) {
        s_prefix = prefix | ((uint32_t)(hi - 1 - x) << shift);
        s_krem = krem - above;
      }
      above += cnt[x];
    }
    __syncthreads();
    prefix = s_prefix;
    krem = s_krem;
    __syncthreads();
  }
  // keys above the threshold, then krem of its ties in ascending u
  const uint32_t tau = prefix;
  int carry_sel = 0, carry_tie = 0;
  for (int u0 = 0; u0 < L; u0 += kSelThreads) {
    const int u = u0 + tid;
    const uint32_t key = u < L ? keys[u] : 0u;
    const bool gt = u < L && key > tau;
    const bool tie = u < L && key == tau;
    int tot_tie = 0;
    const int tie_before = carry_tie + block_excl_scan(tie ? 1 : 0, s_warp, tot_tie);
    const bool sel = gt || (tie && tie_before < krem);
    int tot_sel = 0;
    const int pos = carry_sel + block_excl_scan(sel ? 1 : 0, s_warp, tot_sel);
    if (sel && pos < Lc) out[pos] = u;
    carry_tie += tot_tie;
    carry_sel += tot_sel;
  }
}

// kc[b, c, h, :] = k[b, cols[b, h, c], h / g, :] and likewise v, 16 bytes per thread.
__global__ void col_gather_kernel(const uint8_t* __restrict__ k, const uint8_t* __restrict__ v,
                                  ColArgs c, const int32_t* __restrict__ cols, int Lc,
                                  int esize, uint8_t* __restrict__ kc, uint8_t* __restrict__ vc) {
  const int per = 16 / esize;  // elements per 16 bytes
  const int chunks = c.d / per;
  const int64_t n = (int64_t)c.B * Lc * c.H * chunks;
  const int g = c.H / c.Hkv;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n;
       x += (int64_t)gridDim.x * blockDim.x) {
    const int ch = (int)(x % chunks);
    const int h = (int)((x / chunks) % c.H);
    const int cc = (int)((x / ((int64_t)chunks * c.H)) % Lc);
    const int b = (int)(x / ((int64_t)chunks * c.H * Lc));
    const int u = cols[((int64_t)b * c.H + h) * Lc + cc];
    const int64_t src_k = (b * c.ks[0] + (int64_t)u * c.ks[1] + (h / g) * c.ks[2]) * esize +
                          (int64_t)ch * 16;
    const int64_t src_v = (b * c.vs[0] + (int64_t)u * c.vs[1] + (h / g) * c.vs[2]) * esize +
                          (int64_t)ch * 16;
    const int64_t dst = (((int64_t)b * Lc + cc) * c.H + h) * (int64_t)c.d * esize + (int64_t)ch * 16;
    *reinterpret_cast<uint4*>(kc + dst) = __ldg(reinterpret_cast<const uint4*>(k + src_k));
    *reinterpret_cast<uint4*>(vc + dst) = __ldg(reinterpret_cast<const uint4*>(v + src_v));
  }
}

}  // namespace

size_t col_partial_bytes(const sdl_shape& s) {
  return sizeof(float2) * (size_t)s.B * s.H * (s.L / s.block) * col_groups(s.L);
}

cudaError_t launch_col_scores(const void* k, const sdl_shape& s, float scale, const float* qbar,
                              float2* part, float2* stats, float* S, cudaStream_t st) {
  ColArgs c;
  fill_col_args(c, s, scale);
  const size_t smem1 = col_smem_bytes(s.d), smem2 = smem1 + kColSumExtra;
  const int ngroups = col_groups(s.L);
  const dim3 g1(ngroups, (c.nb + kGR - 1) / kGR, s.B * s.H), g2((s.L + kGK - 1) / kGK, s.B * s.H);
  static std::atomic<bool> attr_set[64];  // per device; the size needed is at most this
  cudaError_t ae = once_per_device(attr_set, [] {
    const int most = (int)(col_smem_bytes(128) + kColSumExtra);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(col_stats_kernel<__nv_bfloat16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, most)) ||
        (e = cudaFuncSetAttribute(col_sum_kernel<__nv_bfloat16>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, most)) ||
        (e = cudaFuncSetAttribute(col_stats_kernel<float>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, most)) ||
        (e = cudaFuncSetAttribute(col_sum_kernel<float>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, most)))
      return e;
    return cudaSuccess;
  });
  if (ae != cudaSuccess) return ae;
  const int rows = s.B * s.H * c.nb;
  if (s.dtype == SDL_BF16) {
    col_stats_kernel<__nv_bfloat16><<<g1, kGT, smem1, st>>>(
        qbar, static_cast<const __nv_bfloat16*>(k), c, part);
  } else {
    col_stats_kernel<float><<<g1, kGT, smem1, st>>>(qbar, static_cast<const float*>(k), c, part);
  }
  col_combine_kernel<<<(rows + 255) / 256, 256, 0, st>>>(part, rows, ngroups, stats);
  if (s.dtype == SDL_BF16) {
    col_sum_kernel<__nv_bfloat16><<<g2, kGT, smem2, st>>>(
        qbar, static_cast<const __nv_bfloat16*>(k), c, stats, S);
  } else {
    col_sum_kernel<float><<<g2, kGT, smem2, st>>>(qbar, static_cast<const float*>(k), c, stats,
                                                   S);
  }
  return cudaGetLastError();
}

cudaError_t launch_col_select(const float* S, int BH, int L, int Lc, int32_t* cols,
                              cudaStream_t st) {
  col_select_kernel<<<BH, kSelThreads, 0, st>>>(S, L, Lc, cols);
  return cudaGetLastError();
}

cudaError_t launch_col_gather(const void* k, const void* v, const sdl_shape& s,
                              const int32_t* cols, int Lc, void* kc, void* vc, cudaStream_t st) {
  ColArgs c;
  fill_col_args(c, s, 0.f);
  const int esize = s.dtype == SDL_BF16 ? 2 : 4;
  const int64_t n = (int64_t)s.B * Lc * s.H * (s.d * esize / 16);
  int64_t grid = (n + 255) / 256;
  if (grid > 148 * 16) grid = 148 * 16;
  col_gather_kernel<<<(unsigned)grid, 256, 0, st>>>(
      static_cast<const uint8_t*>(k), static_cast<const uint8_t*>(v), c, cols, Lc, esize,
      static_cast<uint8_t*>(kc), static_cast<uint8_t*>(vc));
  return cudaGetLastError();
}

}  // namespace sdl
