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
//   warps 2-9   softmax in two warpgroups: each thread one query row (its
//               TMEM lane) and one 64-column half of the step; online softmax
//               in the log2 domain with the running max raised only when it
//               grows by more than 8 (a factor 256), O rescaled in TMEM only
//               then; P written back as bf16 over its S columns and the row
//               sum taken over those rounded weights.
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
constexpr int kThreads = 352;   // 11 warps
constexpr int kVWarp = 10;      // V producer
constexpr int kBox = 64 * 128;  // bytes of one 64-row x 64-column bf16 box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kPolyPer8 = 2;  // of every 8 weights, how many take exp2_poly (FMA pipe)

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
  uint64_t kempty[kStages];  // K slot free: its S product completed
  uint64_t vempty[kStages];  // V slot free: its PV product completed
  uint64_t s[2];
  uint64_t p[2];
  uint64_t o;
  uint64_t done;
  uint64_t soft;  // barrier of the 256 softmax threads
};

__device__ __forceinline__ void raise_timeout(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicOr(status, kDevTimeout);
}

template <int D, bool kLse>
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
  __shared__ float sh_max[2][2][kBM];  // [step parity][group][row] tile maxima
  __shared__ float sh_sum[2][2][kBM];  // [rounded, unrounded][group][row] row sums

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
        mbar_init(&bars.kempty[s], 1);
        mbar_init(&bars.vempty[s], 1);
      }
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bars.s[s], 1);
        mbar_init(&bars.p[s], 8);  // one elected arrival per softmax warp
      }
      mbar_init(&bars.o, 1);
      mbar_init(&bars.done, 1);
      mbar_init(&bars.soft, 8);  // the 8 softmax warps
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

  if (warp == 0 || warp == kVWarp) {
    // --------------------------------------------------------- producers
    // Warp 0 loads Q once and then the K sub-blocks of every step, warp
    // kVWarp the V sub-blocks: two issuing threads, two independent rings
    // (one thread's tensor-copy issue rate alone falls short of a step).
    const bool isk = warp == 0;
    uint64_t* full = isk ? bars.kfull : bars.vfull;
    uint64_t* empty = isk ? bars.kempty : bars.vempty;
    const CUtensorMap* tm = isk ? &tmk : &tmv;
    uint8_t* ring = dsm + (isk ? Lay::kOffK : Lay::kOffV);
    if (lane == 0 && n_steps > 0) {
      prefetch_tensormap(tm);
      if (isk) {
        prefetch_tensormap(&tmq);
        uint8_t* sq = dsm + Lay::kOffQ;
        mbar_arrive_expect_tx(&bars.q, Lay::kQBytes);
        for (int c = 0; c < Lay::kChunks; ++c)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(sq + c * Lay::kChunkRowsQ + s * kBox, &tmq, &bars.q, c * 64, t0 + 64 * s,
                        h, b);
      }
      int done_steps = 0;
      for (int st = 0; st < n_steps; ++st) {
        const int stage = st % kStages;
        if (st >= kStages &&
            !mbar_wait(&empty[stage], ((st / kStages) - 1) & 1, &abort_sh, a.status,
                       kWaitLimitNs)) {
          raise_timeout(&abort_sh, a.status);
          break;
        }
        const uint32_t e0 = ent[2 * st];
        const uint32_t e1 = (2 * st + 1 < n_ent) ? ent[2 * st + 1] : e0;
        const int sub0 = (int)(e0 & 0xFFFFu), sub1 = (int)(e1 & 0xFFFFu);
        uint8_t* dst = ring + stage * Lay::kKVBytes;
        mbar_arrive_expect_tx(&full[stage], Lay::kKVBytes);
        for (int c = 0; c < Lay::kChunks; ++c)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, tm, &full[stage], c * 64,
                        (s ? sub1 : sub0) * kSubBlock, kh, b);
        done_steps = st + 1;
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      volatile int no_abort = 0;
      if (isk && !mbar_wait(&bars.q, 0, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
      for (int st = (done_steps > kStages ? done_steps - kStages : 0); st < done_steps; ++st)
        if (!mbar_wait(&full[st % kStages], (st / kStages) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
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
        tc_commit(&bars.kempty[stage]);
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
          // P elements [16 kk, 16 kk + 16): columns 64 (kk / 4) + 8 (kk % 4)
          mma_bf16_ts(tmem + kColO, pcol + 64 * (kk / 4) + 8 * (kk % 4), bd, idPV,
                      (st > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars.vempty[stage]);
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
    // Two warpgroups: group g owns key columns [64 g, 64 g + 64) of each S
    // row (key sub-block g of the step) and columns [64 g, 64 g + 64) of O.
    // The two threads of a row swap their tile maxima through shared memory
    // once per step.  Each group writes its half of P (bf16 pairs) over the
    // first 32 of its own 64 S columns, so neither group overwrites S the
    // other may still read.
    const int grp = (warp - 2) / 4;
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = a.scale_log2;
    float m = -INFINITY;  // running max (log2 units) used as the exponent reference
    float l = 0.f;        // this half-row's sum of the bf16-rounded weights
    float lx = 0.f;       // this half-row's sum of the unrounded weights (LSE only)
    uint32_t soft_uses = 0;
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
      const bool keep = ((grp ? e1 : e0) >> (16 + half)) & 1u;
      const uint32_t scol = trow + (buf ? kColS1 : kColS0);
      float sv[64];
      {
        uint32_t r[64];
        tmem_ld32(scol + 64 * grp, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(scol + 64 * grp + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 64; ++x) sv[x] = keep ? __uint_as_float(r[x]) * sl2 : -INFINITY;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int x = 0; x < 64; x += 2) mt = fmaxf(mt, fmaxf(sv[x], sv[x + 1]));
      sh_max[st & 1][grp][row] = mt;
      if (!(ok = group_sync(&bars.soft, soft_uses, &abort_sh, a.status, kWaitLimitNs))) break;
      mt = fmaxf(mt, sh_max[st & 1][grp ^ 1][row]);
      const bool raise = mt > m + 8.0f;
      if (__any_sync(0xffffffffu, raise)) {
        if (st > 0) {
          // O must hold every product issued so far before it is rescaled;
          // PV(st-2) is complete (S(st) was committed after it), PV(st-1) may
          // not be, so this wait is unambiguous.
          ok = mbar_wait(&bars.o, (st - 1) & 1, &abort_sh, a.status, kWaitLimitNs);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = raise ? ex2_approx(m - mt) : 1.0f;
          l *= alpha;
          lx *= alpha;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t ov[32];
            const uint32_t oc = trow + kColO + (D / 2) * grp + c * 32;
            tmem_ld32(oc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
            tmem_st32(oc, ov);
          }
          tmem_wait_st();
        }
        if (raise) m = mt;
      }
      // P = exp2(S * scale * log2e - m) on a kept half, 0 otherwise (a kept
      // half always has a finite reference here: its own maximum raised it)
      if (keep) {
#pragma unroll
        for (int x = 0; x < 64; x += 2) {
          if ((x & 7) < 8 - kPolyPer8) {
            sv[x] = ex2_approx(sv[x] - m);
            sv[x + 1] = ex2_approx(sv[x + 1] - m);
          } else {
            const float2 e = exp2_poly2(sv[x] - m, sv[x + 1] - m);
            sv[x] = e.x;
            sv[x + 1] = e.y;
          }
        }
      } else {
#pragma unroll
        for (int x = 0; x < 64; ++x) sv[x] = 0.f;
      }
      // bf16 pairs of P over the S columns; l sums the rounded weights
      float rs = 0.f, rx = 0.f;
      uint32_t pw[32];
#pragma unroll
      for (int x = 0; x < 64; x += 2) {
        __nv_bfloat162 pk = __floats2bfloat162_rn(sv[x], sv[x + 1]);
        const uint32_t u = *reinterpret_cast<uint32_t*>(&pk);
        rs += __uint_as_float(u << 16) + __uint_as_float(u & 0xFFFF0000u);
        if constexpr (kLse) rx += sv[x] + sv[x + 1];
        pw[x / 2] = u;
      }
      l += rs;
      lx += rx;
      // P of this half goes over this half's own S columns [64 grp, 64 grp + 32)
      // (never over columns the other group may still read)
      tmem_st32(scol + 64 * grp, pw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p[buf]);
    }
    // ------------------------------------------------------- epilogue
    const int t = t0 + row;
    if (ok && n_steps > 0) {
      // full-row sums from the two halves
      sh_sum[0][grp][row] = l;
      sh_sum[1][grp][row] = lx;
      ok = group_sync(&bars.soft, soft_uses, &abort_sh, a.status, kWaitLimitNs);
      l += sh_sum[0][grp ^ 1][row];
      lx += sh_sum[1][grp ^ 1][row];
    }
    if (!ok) {
      raise_timeout(&abort_sh, a.status);
    } else if (n_steps == 0) {
      if (t < a.L) {
        __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                            (int64_t)t * a.os[1] + h * a.os[2] + (D / 2) * grp;
        for (int c = 0; c < D / 2; c += 8) *reinterpret_cast<uint4*>(op + c) = make_uint4(0, 0, 0, 0);
        if (a.lse && grp == 0) a.lse[((int64_t)b * a.H + h) * a.L + t] = -INFINITY;
      }
    } else if (__all_sync(0xffffffffu,
                          mbar_wait(&bars.done, 0, &abort_sh, a.status, kWaitLimitNs))) {
      // (bars.done completes once, after every MMA of the tile: with the lazy
      //  waits above, the last two products may still be running here)
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                          (int64_t)t * a.os[1] + h * a.os[2] + (D / 2) * grp;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[32];
        tmem_ld32(trow + kColO + (D / 2) * grp + c * 32, ov);
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
      if (a.lse && grp == 0 && t < a.L)
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

template <int D, bool kLse>
static cudaError_t launch_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, cudaStream_t st) {
  using Lay = Layout<D>;
  dim3 grid((a.L + kBM - 1) / kBM, a.H, a.B);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, kLse>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D, kLse><<<grid, kThreads, Lay::kSmem, st>>>(*tq, *tk, *tv, a);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, cudaStream_t st) {
  if (a.d == 128)
    return a.lse ? launch_tc<128, true>(a, tq, tk, tv, st) : launch_tc<128, false>(a, tq, tk, tv, st);
  return a.lse ? launch_tc<64, true>(a, tq, tk, tv, st) : launch_tc<64, false>(a, tq, tk, tv, st);
}

}  // namespace sdl
