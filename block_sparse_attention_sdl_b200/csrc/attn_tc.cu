// bf16 block-sparse / dense attention on sm_100a tensor cores.
//
// The fused IO-aware block-sparse kernel of the Step-dLLM abstract,
// re-designed for Blackwell: each CTA owns a 128-row query tile of one head
// and walks the kept key blocks of its rows, two 64-token sub-blocks per step.
//
//   warp 0      TMA producer: Q once, then K and V sub-blocks of each step
//               (128-byte-swizzled 64x64 boxes) into a 2-stage ring.
//   warp 1      TMEM allocator and MMA issuer (one thread):
//                 S = Q K^T   tcgen05.mma kind::f16, A and B from shared memory,
//                             M=128, N=128, fp32 accumulator in TMEM;
//                 O += P V    A = P (bf16) from TMEM, B = V from shared memory
//                             (N-major), M=128, N=d.
//   warps 2-5   softmax: one thread per query row (its TMEM lane), online
//               softmax in the log2 domain with the running max raised only
//               when it grows by more than 8 (a factor 256), O rescaled in
//               TMEM only then; P written back as bf16 over its S columns and
//               the row sum taken over those rounded weights.
//               Epilogue: O / l rounded to bf16, LSE.
//
// With 64-token blocks a 128-row tile covers two query blocks; the kernel
// walks the union of their kept lists and masks, per 64x64 quadrant, the
// key sub-blocks a query block did not keep.  With 128-token blocks both
// halves share one list.  Dense attention is the same walk over every
// sub-block.
//
// TMEM columns: S/P buffers at 0 and 128, O at 256 (512 allocated).
// Every mbarrier wait is bounded; on timeout the CTA raises the device
// status word, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace sdl {
namespace {

constexpr int kBM = 128;        // query rows per CTA
constexpr int kBN = 128;        // key rows per step
constexpr int kStages = 2;      // K/V ring depth
constexpr int kMaxSub = 1024;   // 64-token sub-blocks per sequence (L <= 65536)
constexpr int kThreads = 192;   // 6 warps
constexpr int kBox = 64 * 128;  // bytes of one 64-row x 64-column bf16 box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;                  // 128-byte column chunks
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;            // one stage of K (or V)
  static constexpr int kChunkRowsQ = kBM * 128;           // bytes per Q column chunk
  static constexpr int kChunkRowsKV = kBN * 128;          // bytes per K/V column chunk
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kBytes = kOffV + kStages * kKVBytes;
  static constexpr int kSmem = kBytes + 1024;             // + alignment slack
};

struct Bars {
  uint64_t q;
  uint64_t kfull[kStages];
  uint64_t vfull[kStages];
  uint64_t kvempty[kStages];
  uint64_t s[2];
  uint64_t p[2];
  uint64_t o;
  uint64_t done;
};

__device__ __forceinline__ void raise_timeout(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicOr(status, kDevTimeout);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, AttnArgs a) {
  using Lay = Layout<D>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                            ~(uintptr_t)1023);
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  __shared__ uint32_t ent[kMaxSub];  // sub-block | keep bits << 16
  __shared__ uint32_t bmask[2][kMaxSub / 32];
  __shared__ int n_ent_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int t0 = blockIdx.x * kBM;
  const int kh = h / (a.H / a.Hkv);
  const int nsub = a.L / kSubBlock;

  // ------------------------------------------------------------ set-up
  if (warp == 0) {
    // Kept 64-token key sub-blocks for the two query halves, as bitmaps.
    for (int w = lane; w < kMaxSub / 32; w += 32) bmask[0][w] = bmask[1][w] = 0;
    __syncwarp();
    if (a.row_ptr == nullptr) {
      for (int s = lane; s < nsub; s += 32) {
        atomicOr(&bmask[0][s / 32], 1u << (s % 32));
        atomicOr(&bmask[1][s / 32], 1u << (s % 32));
      }
    } else {
      const int per = a.block / kSubBlock;  // sub-blocks per block: 1 or 2
      const int rows_in_tile = a.block == 64 ? 2 : 1;
      for (int rr = 0; rr < rows_in_tile; ++rr) {
        const int i = t0 / a.block + rr;
        if (i >= a.nb) break;
        const int64_t r = ((int64_t)b * a.H + h) * a.nb + i;
        const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
        for (int x = beg + lane; x < end; x += 32) {
          const int j = a.col_idx[x];
          const bool bad_range = j < 0 || j >= a.nb;
          if (bad_range || (x > beg && a.col_idx[x - 1] >= j)) atomicOr(a.status, kDevBadMask);
          if (bad_range) continue;
          for (int u = 0; u < per; ++u) {
            const int s = j * per + u;
            if (a.block == 64) {
              atomicOr(&bmask[rr][s / 32], 1u << (s % 32));
            } else {
              atomicOr(&bmask[0][s / 32], 1u << (s % 32));
              atomicOr(&bmask[1][s / 32], 1u << (s % 32));
            }
          }
        }
      }
    }
    __syncwarp();
    // Ascending union with per-half keep bits: lane w handles bitmap word w.
    const uint32_t w0 = bmask[0][lane], w1 = bmask[1][lane];
    const uint32_t wu = w0 | w1;
    const int c = __popc(wu);
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int pos = incl - c;
    for (uint32_t m = wu; m; m &= m - 1) {
      const int bit = __ffs(m) - 1;
      const uint32_t keep = ((w0 >> bit) & 1u) | (((w1 >> bit) & 1u) << 1);
      ent[pos++] = (uint32_t)(lane * 32 + bit) | (keep << 16);
    }
    if (lane == 31) n_ent_sh = incl;
  } else if (warp == 1) {
    if (lane == 0) {
      mbar_init(&bars.q, 1);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&bars.kfull[s], 1);
        mbar_init(&bars.vfull[s], 1);
        mbar_init(&bars.kvempty[s], 1);
      }
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bars.s[s], 1);
        mbar_init(&bars.p[s], 128);
      }
      mbar_init(&bars.o, 1);
      mbar_init(&bars.done, 1);
      abort_sh = 0;
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int n_ent = n_ent_sh;
  const int n_steps = (n_ent + 1) / 2;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0 && n_steps > 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      uint8_t* sq = dsm + Lay::kOffQ;
      mbar_arrive_expect_tx(&bars.q, Lay::kQBytes);
      for (int c = 0; c < Lay::kChunks; ++c)
        for (int s = 0; s < 2; ++s)
          tma_load_4d(sq + c * Lay::kChunkRowsQ + s * kBox, &tmq, &bars.q, c * 64, t0 + 64 * s, h,
                      b);
      int issued[kStages] = {0};
      for (int st = 0; st < n_steps; ++st) {
        const int stage = st % kStages;
        if (st >= kStages) {
          if (!mbar_wait(&bars.kvempty[stage], ((st / kStages) - 1) & 1, &abort_sh, a.status, kWaitLimitNs)) {
            raise_timeout(&abort_sh, a.status);
            break;
          }
        }
        const uint32_t e0 = ent[2 * st];
        const uint32_t e1 = (2 * st + 1 < n_ent) ? ent[2 * st + 1] : e0;
        const int sub[2] = {(int)(e0 & 0xFFFFu), (int)(e1 & 0xFFFFu)};
        uint8_t* sk = dsm + Lay::kOffK + stage * Lay::kKVBytes;
        uint8_t* sv = dsm + Lay::kOffV + stage * Lay::kKVBytes;
        mbar_arrive_expect_tx(&bars.kfull[stage], Lay::kKVBytes);
        for (int c = 0; c < Lay::kChunks; ++c)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(sk + c * Lay::kChunkRowsKV + s * kBox, &tmk, &bars.kfull[stage], c * 64,
                        sub[s] * kSubBlock, kh, b);
        mbar_arrive_expect_tx(&bars.vfull[stage], Lay::kKVBytes);
        for (int c = 0; c < Lay::kChunks; ++c)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(sv + c * Lay::kChunkRowsKV + s * kBox, &tmv, &bars.vfull[stage], c * 64,
                        sub[s] * kSubBlock, kh, b);
        ++issued[stage];
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      volatile int no_abort = 0;
      if (!mbar_wait(&bars.q, 0, &no_abort, nullptr, kWaitLimitNs)) atomicOr(a.status, kDevTimeout);
      for (int s = 0; s < kStages; ++s) {
        if (issued[s] == 0) continue;
        const uint32_t par = (issued[s] - 1) & 1;
        if (!mbar_wait(&bars.kfull[s], par, &no_abort, nullptr, kWaitLimitNs)) atomicOr(a.status, kDevTimeout);
        if (!mbar_wait(&bars.vfull[s], par, &no_abort, nullptr, kWaitLimitNs)) atomicOr(a.status, kDevTimeout);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kBM, D, true);
      const uint32_t q_base = smem_u32(dsm + Lay::kOffQ);
      const uint32_t k_base = smem_u32(dsm + Lay::kOffK);
      const uint32_t v_base = smem_u32(dsm + Lay::kOffV);
      bool ok = mbar_wait(&bars.q, 0, &abort_sh, a.status, kWaitLimitNs);
      auto issue_s = [&](int st) -> bool {
        const int stage = st % kStages;
        if (!mbar_wait(&bars.kfull[stage], (st / kStages) & 1, &abort_sh, a.status, kWaitLimitNs))
          return false;
        tc_fence_after();
        const uint32_t kb = k_base + stage * Lay::kKVBytes;
        const uint32_t dcol = tmem + ((st & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk % 4) * 32;  // 16 bf16 of K inside the swizzle atom
          const uint64_t ad = smem_desc_sw128(q_base + (kk / 4) * Lay::kChunkRowsQ + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kb + (kk / 4) * Lay::kChunkRowsKV + off, 16, 1024);
          mma_bf16_ss(dcol, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars.s[st & 1]);
        return true;
      };
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
      for (int st = 0; ok && st < n_steps; ++st) {
        if (st + 1 < n_steps && !(ok = issue_s(st + 1))) break;
        if (!(ok = mbar_wait(&bars.p[st & 1], (st >> 1) & 1, &abort_sh, a.status, kWaitLimitNs))) break;
        const int stage = st % kStages;
        if (!(ok = mbar_wait(&bars.vfull[stage], (st / kStages) & 1, &abort_sh, a.status, kWaitLimitNs)))
          break;
        tc_fence_after();
        const uint32_t vb = v_base + stage * Lay::kKVBytes;
        const uint32_t pcol = tmem + ((st & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(vb + kk * 16 * 128, Lay::kChunkRowsKV, 1024);
          mma_bf16_ts(tmem + kColO, pcol + kk * 8, bd, idPV, (st > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars.kvempty[stage]);
        tc_commit(&bars.o);
      }
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Every MMA issued above completes before TMEM is released.
      tc_commit(&bars.done);
      volatile int no_abort = 0;
      if (!mbar_wait(&bars.done, 0, &no_abort, nullptr, kWaitLimitNs)) atomicOr(a.status, kDevTimeout);
    }
  } else {
    // --------------------------------------------------------- softmax
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = a.scale_log2;
    float m = -INFINITY;  // running max (log2 units) used as the exponent reference
    float l = 0.f;        // sum of the bf16-rounded weights (normalises O)
    float lx = 0.f;       // sum of the unrounded weights (for the LSE)
    bool ok = true;
    for (int st = 0; st < n_steps; ++st) {
      const int buf = st & 1;
      ok = mbar_wait(&bars.s[buf], (st >> 1) & 1, &abort_sh, a.status, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t e0 = ent[2 * st];
      const uint32_t e1 = (2 * st + 1 < n_ent) ? ent[2 * st + 1] : (e0 & 0xFFFFu);
      const bool v0 = (e0 >> (16 + half)) & 1u;
      const bool v1 = (e1 >> (16 + half)) & 1u;
      const uint32_t scol = trow + (buf ? kColS1 : kColS0);
      uint32_t sr[4][32];
      tmem_ld32(scol + 0, sr[0]);
      tmem_ld32(scol + 32, sr[1]);
      tmem_ld32(scol + 64, sr[2]);
      tmem_ld32(scol + 96, sr[3]);
      tmem_wait_ld();
      float mt = -INFINITY;
      if (v0) {
#pragma unroll
        for (int x = 0; x < 32; ++x) mt = fmaxf(mt, fmaxf(__uint_as_float(sr[0][x]), __uint_as_float(sr[1][x])));
      }
      if (v1) {
#pragma unroll
        for (int x = 0; x < 32; ++x) mt = fmaxf(mt, fmaxf(__uint_as_float(sr[2][x]), __uint_as_float(sr[3][x])));
      }
      mt *= sl2;
      const bool raise = mt > m + 8.0f;
      if (st > 0) {
        ok = mbar_wait(&bars.o, (st - 1) & 1, &abort_sh, a.status, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // tcgen05.ld/st are warp-collective: the warp rescales together, alpha = 1
        // on rows whose reference max stays.
        if (__any_sync(0xffffffffu, raise)) {
          const float alpha = raise ? ex2_approx(m - mt) : 1.0f;
          l *= alpha;
          lx *= alpha;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(trow + kColO + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
            tmem_st32(trow + kColO + c * 32, ov);
          }
        }
      }
      if (raise) m = mt;
      // P = exp2(S * scale * log2e - m) on kept quadrants, 0 elsewhere; bf16 pairs.
      float rs = 0.f, rx = 0.f;
      uint32_t pw[2][32];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const bool keep = g < 2 ? v0 : v1;
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          float p0 = 0.f, p1 = 0.f;
          if (keep) {
            p0 = ex2_approx(fmaf(__uint_as_float(sr[g][x]), sl2, -m));
            p1 = ex2_approx(fmaf(__uint_as_float(sr[g][x + 1]), sl2, -m));
          }
          // l sums the bf16-rounded weights that the PV product uses, so the
          // normalisation matches the numerator exactly
          __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
          const float2 pr = __bfloat1622float2(pk);
          rs += pr.x + pr.y;
          rx += p0 + p1;
          pw[g >> 1][(g & 1) * 16 + x / 2] = *reinterpret_cast<uint32_t*>(&pk);
        }
      }
      l += rs;
      lx += rx;
      tmem_st32(scol + 0, pw[0]);
      tmem_st32(scol + 32, pw[1]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars.p[buf]);
    }
    // ------------------------------------------------------- epilogue
    const int t = t0 + row;
    if (!ok) {
      raise_timeout(&abort_sh, a.status);
    } else if (n_steps == 0) {
      if (t < a.L) {
        __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                            (int64_t)t * a.os[1] + h * a.os[2];
        for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(op + c) = make_uint4(0, 0, 0, 0);
        if (a.lse) a.lse[((int64_t)b * a.H + h) * a.L + t] = -INFINITY;
      }
    } else if (__all_sync(0xffffffffu,
                          mbar_wait(&bars.o, (n_steps - 1) & 1, &abort_sh, a.status, kWaitLimitNs))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                          (int64_t)t * a.os[1] + h * a.os[2];
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(trow + kColO + c * 32, ov);
        tmem_wait_ld();
        if (t < a.L) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(ov[2 * x]) * inv,
                                                     __uint_as_float(ov[2 * x + 1]) * inv);
            pk[x] = *reinterpret_cast<uint32_t*>(&v);
          }
          uint4* dst = reinterpret_cast<uint4*>(op + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      if (a.lse && t < a.L)
        a.lse[((int64_t)b * a.H + h) * a.L + t] =
            lx > 0.f ? (m + log2f(lx)) * 0.69314718055994531f : -INFINITY;
    } else {
      raise_timeout(&abort_sh, a.status);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, cudaStream_t st) {
  dim3 grid((a.L + kBM - 1) / kBM, a.H, a.B);
  if (a.d == 128) {
    using Lay = Layout<128>;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<128><<<grid, kThreads, Lay::kSmem, st>>>(*tq, *tk, *tv, a);
  } else {
    using Lay = Layout<64>;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<64><<<grid, kThreads, Lay::kSmem, st>>>(*tq, *tk, *tv, a);
  }
  return cudaGetLastError();
}

}  // namespace sdl
