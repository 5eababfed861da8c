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
// A 16-byte read-only load; kStream: no L1 allocation and a 256-byte L2
// prefetch (each token's 512-byte chunk is read once).
template <bool kStream>
__device__ __forceinline__ uint4 load16(const void* p) {
  if constexpr (kStream) {
    uint4 u;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                 : "l"(p));
    return u;
  } else {
    return __ldg(reinterpret_cast<const uint4*>(p));
  }
}

// Pooling work item `it` (Q items first, then K; each item: batch element b,
// block i, chunk of 32 lanes x 16 bytes of the contiguous (h, d) plane): this
// warp sums its elements over the block's tokens with independent 16-byte
// loads, then writes the means.
template <typename T, int kUnroll, bool kStream>
__device__ __forceinline__ void pool_item(const PoolTensor& tq, const PoolTensor& tk, int64_t it,
                                          int64_t items_q, int nb, int d, int bs, int lane) {
  constexpr int V = Vec<T>::N;
  const bool isq = it < items_q;
  const PoolTensor& tx = isq ? tq : tk;
  const int64_t r = isq ? it : it - items_q;
  const int chunk = (int)(r % tx.chunks);
  const int i = (int)((r / tx.chunks) % nb);
  const int b = (int)(r / ((int64_t)tx.chunks * nb));
  const int e = (chunk * 32 + lane) * V;  // element of the (h, d) plane
  if (e >= tx.Hx * d) return;
  const int h = e / d, c = e % d;
  const T* base =
      reinterpret_cast<const T*>(tx.x) + b * tx.s0 + h * tx.s2 + c + (int64_t)i * bs * tx.s1;
  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
#pragma unroll kUnroll
  for (int t = 0; t < bs; ++t) {
    const uint4 u = load16<kStream>(base + (int64_t)t * tx.s1);
    Vec<T>::add(acc, u);
  }
  const float inv = 1.0f / (float)bs;
  float* dst = tx.out + (((int64_t)b * tx.Hx + h) * nb + i) * d + c;
#pragma unroll
  for (int v = 0; v < V; v += 4)
    *reinterpret_cast<float4*>(dst + v) =
        make_float4(acc[v] * inv, acc[v + 1] * inv, acc[v + 2] * inv, acc[v + 3] * inv);
}

// Every pooling item, spread over the warps of blocks bx of nbx.
template <typename T, int kUnroll = 16, bool kStream = false>
__device__ __forceinline__ void pool_body(PoolTensor tq, PoolTensor tk, int B, int L, int d,
                                          int bs, int64_t bx, int64_t nbx) {
  const int nb = L / bs;
  const int64_t items_q = (int64_t)B * nb * tq.chunks;
  const int64_t items = items_q + (int64_t)B * nb * tk.chunks;
  const int64_t wpb = blockDim.x / 32;  // warps per block
  for (int64_t it = bx * wpb + threadIdx.x / 32; it < items; it += nbx * wpb)
    pool_item<T, kUnroll, kStream>(tq, tk, it, items_q, nb, d, bs, threadIdx.x % 32);
}

constexpr int kTI = 16;   // query blocks per item (the tensor-core tile's 16 rows)
constexpr int kTJ = 128;  // key blocks per shared-memory tile (8 or 16 per warp)
constexpr int kScoreThreads = 256;

// x = hi + lo with hi = tf32(x) (round to nearest) and lo = tf32(x - hi).
__device__ __forceinline__ void tf32_split(float x, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  const float r = x - __uint_as_float(hi);
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}

// c (16 x 8, fp32) += a (16 x 8, tf32, row-major) * b (8 x 8, tf32, column-major).
__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

inline size_t score_smem_bytes(int nb, int d) {
  return sizeof(float) * ((size_t)(kTI + kTJ) * (d + 4) + (size_t)kTI * nb);
}

// `rows` rows of D floats from global `src` (row `r0` first, rows past `n`
// zero) into shared `dst` with row pitch D + 4, by asynchronous 16-byte copies
// (all in flight at once); the caller waits with cp.async.wait_all and a
// block barrier.
template <int D, int NT>
__device__ __forceinline__ void stage_rows(float* dst, const float* __restrict__ src, int r0,
                                           int rows, int n, int tid) {
  constexpr int d4 = D / 4, dp = D + 4;
  const int total = rows * d4;
  for (int x = tid; x < total; x += NT) {
    const int r = x / d4, c = (x % d4) * 4;
    float* d = dst + r * dp + c;
    if (r0 + r < n) {
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                       static_cast<uint32_t>(__cvta_generic_to_shared(d))),
                   "l"(src + (int64_t)(r0 + r) * D + c)
                   : "memory");
    } else {
      *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}
__device__ __forceinline__ void stage_wait() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Item (query-block tile bx, head h, batch element b) on a block of at least
// NT threads (256 or 512; the first NT work, any further ones only join its
// barriers); shared memory `sm` of score_smem_bytes(nb, D):
//   qs [kTI][D+4], ks [kTJ][D+4], z [kTI][nb] floats.
// Every score is computed by the same arithmetic for either NT.
template <int D, int NT = kScoreThreads, bool kKeep = false>
__device__ __forceinline__ void score_body_d(const float* __restrict__ qbar,
                                             const float* __restrict__ kbar,
                                             float* __restrict__ scores, int H, int Hkv, int nb,
                                             float scale, int bx, int h, int b, float* sm) {
  constexpr int dp = D + 4;
  float* qs = sm;
  float* ks = qs + kTI * dp;
  float* z = ks + kTJ * dp;
  const int i0 = bx * kTI;
  const int kh = h / (H / Hkv);
  const float* qsrc = qbar + (((int64_t)b * H + h) * nb) * D;
  const float* ksrc = kbar + (((int64_t)b * Hkv + kh) * nb) * D;
  static_assert(NT == 256 || NT == 512, "256 or 512 threads");
  constexpr int kTiles = NT == 256 ? 2 : 1;  // 8-key tiles per warp
  const int tid = threadIdx.x;
  const bool act = tid < NT;
  if (act) stage_rows<D, NT>(qs, qsrc, i0, kTI, nb, tid);
  const int ty = tid / 32, tx = tid % 32;
  for (int j0 = 0; j0 < nb; j0 += kTJ) {
    __syncthreads();
    if (act) {
      stage_rows<D, NT>(ks, ksrc, j0, kTJ, nb, tid);
      stage_wait();
    }
    __syncthreads();
    if (!act) continue;
    // Z = Qbar Kbar^T on the tensor cores: warp ty takes key blocks
    // [8 kTiles ty, 8 kTiles (ty + 1)) as 8-column tiles, all 16 query blocks, d in
    // steps of 8 (mma m16n8k8, tf32 in, fp32 accumulate).  Every fp32 operand
    // x is split as hi = tf32(x), lo = tf32(x - hi), and the product taken as
    // hi*hi + hi*lo + lo*hi: about 2^-21 relative per product, fp32-like.
    // Fragment positions (g = lane / 4, t = lane % 4): A rows g, g + 8 and
    // columns t, t + 4; B (= K^T) rows t, t + 4 and column g; C rows g, g + 8
    // and columns 2t, 2t + 1.  Shared-memory rows are D + 4 floats apart, so
    // the 32 lanes' reads hit 32 distinct banks.
    const int g = tx >> 2, t = tx & 3;
    // the hi*hi products and the two cross terms accumulate apart (three
    // independent chains per tile), summed once at the end
    float acc[kTiles][4], accx[kTiles][4];
#pragma unroll
    for (int nt = 0; nt < kTiles; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = accx[nt][e] = 0.f;
    const float* qa = qs + g * dp + t;
    const float* kb = ks + (8 * kTiles * ty + g) * dp + t;
#pragma unroll 4
    for (int k0 = 0; k0 < D; k0 += 8) {
      uint32_t ah[4], al[4];
      tf32_split(qa[k0], ah[0], al[0]);
      tf32_split(qa[8 * dp + k0], ah[1], al[1]);
      tf32_split(qa[k0 + 4], ah[2], al[2]);
      tf32_split(qa[8 * dp + k0 + 4], ah[3], al[3]);
#pragma unroll
      for (int nt = 0; nt < kTiles; ++nt) {
        uint32_t bh[2], bl[2];
        tf32_split(kb[nt * 8 * dp + k0], bh[0], bl[0]);
        tf32_split(kb[nt * 8 * dp + k0 + 4], bh[1], bl[1]);
        mma_tf32(accx[nt], al, bh);
        mma_tf32(acc[nt], ah, bh);
        mma_tf32(accx[nt], ah, bl);
      }
    }
#pragma unroll
    for (int nt = 0; nt < kTiles; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] += accx[nt][e];
#pragma unroll
    for (int nt = 0; nt < kTiles; ++nt) {
      const int j = j0 + 8 * kTiles * ty + 8 * nt + 2 * t;
      if (j < nb) {
        z[g * nb + j] = acc[nt][0] * scale;
        z[(g + 8) * nb + j] = acc[nt][2] * scale;
      }
      if (j + 1 < nb) {
        z[g * nb + j + 1] = acc[nt][1] * scale;
        z[(g + 8) * nb + j + 1] = acc[nt][3] * scale;
      }
    }
  }
  __syncthreads();
  // row softmax: one warp per row; rows of a multiple of 128 blocks are read
  // and written 4 consecutive values per lane
  const int warp = tid / 32, lane = tid % 32;
  if ((nb & 127) == 0) {
    for (int r = act ? warp : kTI; r < kTI; r += NT / 32) {
      if (i0 + r >= nb) break;
      float4* zr = reinterpret_cast<float4*>(z + r * nb);
      const int n4 = nb / 4;
      float m = -INFINITY;
      for (int j = lane; j < n4; j += 32) {
        const float4 v = zr[j];
        m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      for (int j = lane; j < n4; j += 32) {
        float4 v = zr[j];
        v = make_float4(expf(v.x - m), expf(v.y - m), expf(v.z - m), expf(v.w - m));
        zr[j] = v;
        sum += v.x + v.y + v.z + v.w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = 1.0f / sum;
      float4* dst = reinterpret_cast<float4*>(scores + (((int64_t)b * H + h) * nb + (i0 + r)) * nb);
      for (int j = lane; j < n4; j += 32) {
        const float4 v = zr[j];
        const float4 p = make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
        dst[j] = p;
        if (kKeep) zr[j] = p;
      }
    }
    __syncthreads();  // z may be reused by the block's next item
    return;
  }
  for (int r = act ? warp : kTI; r < kTI; r += NT / 32) {
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
    for (int j = lane; j < nb; j += 32) {
      const float p = zr[j] * inv;
      dst[j] = p;
      if (kKeep) zr[j] = p;
    }
  }
  __syncthreads();  // z may be reused by the block's next item
}

// kKeep: the item's normalized rows also stay in shared memory, at
// score_rows_offset(d) floats into `sm`, row r at r * nb (the values written
// to `scores`), until the block's next use of `sm`.
template <bool kKeep = false>
__device__ __forceinline__ void score_body(const float* __restrict__ qbar,
                                           const float* __restrict__ kbar,
                                           float* __restrict__ scores, int H, int Hkv, int nb,
                                           int d, float scale, int bx, int h, int b, float* sm) {
  if (d == 128)
    score_body_d<128, kScoreThreads, kKeep>(qbar, kbar, scores, H, Hkv, nb, scale, bx, h, b, sm);
  else
    score_body_d<64, kScoreThreads, kKeep>(qbar, kbar, scores, H, Hkv, nb, scale, bx, h, b, sm);
}

__host__ __device__ inline size_t score_rows_offset(int d) { return (size_t)(kTI + kTJ) * (d + 4); }

}  // namespace
}  // namespace scimpl
}  // namespace sdl
