// bf16 block-sparse / dense attention on sm_100a tensor cores.
//
// The fused IO-aware block-sparse kernel of the Step-dLLM abstract,
// re-designed for Blackwell.  A work item is a 128-row query tile of one
// head; it walks the kept key blocks of its rows, two 64-token sub-blocks
// (128 keys) per step.  CTAs are persistent (one per SM) and take items from
// a global counter, first come first served (tiles differ in cost by the
// length of their kept lists).  The next item's kept list and Q tile are staged while the
// current one computes, the MMA issuer looks one step ahead across items, and
// two O accumulators let one item's epilogue overlap the next item's products.
//
//   warp 0        K producer: K sub-blocks of every step by TMA
//                 (128-byte-swizzled 64x64 boxes) into a 2-deep ring.
//   warp 10       V producer: the V sub-blocks into their own 2-deep ring (one
//                 issuing thread alone cannot copy a step's K and V in time).
//   warp 11       item producer: the union list of the next item's rows into
//                 one of two shared-memory slots, then its Q tile by TMA into
//                 the matching Q slot.  Items whose lists are empty (only a
//                 caller's mask can have empty rows) are written here as zero
//                 rows and never reach the other warps.
//   warp 1        TMEM allocator and MMA issuer (one thread):
//                   S = Q K^T   tcgen05.mma kind::f16, A and B from shared
//                               memory, M=128, N=128, fp32 into one of two
//                               TMEM S buffers (by step parity);
//                   O += P V    A = P (bf16) from TMEM, B = V from shared
//                               memory (N-major), M=128, N=d, into the
//                               item's TMEM O buffer (by slot).
//   warps 2-9     softmax in two warpgroups: each thread one query row (its
//                 TMEM lane) and one 64-column half of the step; online
//                 softmax in the log2 domain with the running max raised
//                 only when it grows by more than 8 (a factor 256) and O
//                 rescaled in TMEM only then; P written back as bf16 over the
//                 thread's own S columns, the row sum taken over those
//                 rounded weights; 2 of every 8 exponentials on the FMA pipe.
//                 Epilogue per item: O / l rounded to bf16, LSE.
//
// With 64-token blocks a 128-row tile covers two query blocks; the item walks
// the union of their kept lists and masks, per 64x64 quadrant, the key
// sub-blocks a query block did not keep.  With 128-token blocks both halves
// share one list.  Dense attention is the same walk over every sub-block.
//
// TMEM (512 columns): S buffers at columns 0 and 128, O buffers at 256, 384.
// Every mbarrier wait is bounded; on timeout the CTA raises the device
// status word, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "internal.cuh"
#include "ptx.cuh"

namespace sdl {
namespace {

constexpr int kBM = 128;         // query rows per item
constexpr int kBN = 128;         // key rows per step
constexpr int kStages = 2;       // K and V ring depth
constexpr int kSlots = 2;        // item slots: list, Q tile, O accumulator
constexpr int kMaxSub = 1024;    // 64-token sub-blocks per sequence (L <= 65536)
constexpr int kThreads = 384;    // 12 warps
constexpr int kVWarp = 10;       // V producer
constexpr int kItemWarp = 11;    // item producer
constexpr int kSoftWarps = 8;
constexpr int kBox = 64 * 128;   // bytes of one 64-row x 64-column bf16 box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S buffer u at kColS + 128 u
constexpr uint32_t kColO = 256;  // O buffer of slot s at kColO + 128 s
constexpr int kPolyPer8 = 2;     // of every 8 weights, how many take exp2_poly (FMA pipe)

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;           // 128-byte column chunks
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;     // one stage of K (or V)
  static constexpr int kChunkRowsQ = kBM * 128;    // bytes per Q column chunk
  static constexpr int kChunkRowsKV = kBN * 128;   // bytes per K/V column chunk
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kSlots * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kBytes = kOffV + kStages * kKVBytes;
  static constexpr int kSmem = kBytes + 1024;      // + alignment slack
};

struct Bars {
  uint64_t list_full[kSlots];   // slot published by the item producer
  uint64_t list_empty[kSlots];  // slot released by every consumer
  uint64_t q_full[kSlots];
  uint64_t q_empty[kSlots];     // every S product reading the Q slot completed
  uint64_t kfull[kStages], kempty[kStages];  // K slot free once its S product completed
  uint64_t vfull[kStages], vempty[kStages];  // V slot free once its PV product completed
  uint64_t s[2];                // S buffer filled
  uint64_t p[2];                // P written over that S buffer
  uint64_t o;                   // one completion per PV product
  uint64_t o_full[kSlots];      // every product of the slot's item completed
  uint64_t o_empty[kSlots];     // the slot's O read by the epilogue
  uint64_t soft;                // barrier of the softmax warps
  uint64_t done;
};

constexpr int kListConsumers = 3 + kSoftWarps;  // MMA, K and V producers, softmax warps

// One published item: its kept list, sub-block index | keep bits << 16
// (bit 0: query rows 0..63 keep it, bit 1: rows 64..127).
struct Slot {
  int item;  // -1: end of this CTA's schedule
  int n_ent;
  int b, h, t0;
  uint32_t ent[kMaxSub];
};

// Item counters of in-flight launches.  Launch n uses entry n % kSchedRing;
// its CTAs take items with atomicAdd on `next`, and the last CTA to finish
// puts the entry back to zero for a later launch.
constexpr int kSchedRing = 64;
struct Sched {
  unsigned next;
  unsigned finished;
};
__device__ Sched g_sched[kSchedRing];

__device__ __forceinline__ void raise_timeout(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicOr(status, kDevTimeout);
}

// Zero output rows (and -inf LSE) of a 128-row tile whose kept list is empty.
template <int D>
__device__ __forceinline__ void write_empty_tile(const AttnArgs& a, int b, int h, int t0, int lane) {
  for (int r = lane; r < kBM; r += 32) {
    const int t = t0 + r;
    if (t >= a.L) break;
    uint4* op = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                                         (int64_t)t * a.os[1] + h * a.os[2]);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) op[c] = make_uint4(0, 0, 0, 0);
    if (a.lse) a.lse[((int64_t)b * a.H + h) * a.L + t] = -INFINITY;
  }
}

template <int D, bool kLse>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, AttnArgs a, int sched_slot) {
  using Lay = Layout<D>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                            ~(uintptr_t)1023);
  __shared__ Bars bars;
  __shared__ Slot slots[kSlots];
  __shared__ uint32_t bmask[2][kMaxSub / 32];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  __shared__ float sh_max[2][2][kBM];  // [step parity][group][row] tile maxima
  __shared__ float sh_sum[2][2][kBM];  // [rounded, unrounded][group][row] row sums

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = (a.L + kBM - 1) / kBM;
  const int n_items = a.B * a.H * n_qt;

  if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < kSlots; ++s) {
        mbar_init(&bars.list_full[s], 1);
        mbar_init(&bars.list_empty[s], kListConsumers);
        mbar_init(&bars.q_full[s], 1);
        mbar_init(&bars.q_empty[s], 1);
        mbar_init(&bars.o_full[s], 1);
        mbar_init(&bars.o_empty[s], kSoftWarps);
      }
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&bars.kfull[s], 1);
        mbar_init(&bars.kempty[s], 1);
        mbar_init(&bars.vfull[s], 1);
        mbar_init(&bars.vempty[s], 1);
      }
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bars.s[s], 1);
        mbar_init(&bars.p[s], kSoftWarps);  // one elected arrival per softmax warp
      }
      mbar_init(&bars.o, 1);
      mbar_init(&bars.soft, kSoftWarps);
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

  if (warp == kItemWarp) {
    // ====================================================== item producer
    // Takes items from the launch's counter and publishes the non-empty ones,
    // in order, into slots k % kSlots (k = publication ordinal), then the
    // end marker.
    const int nsub = a.L / kSubBlock;
    int qiss0 = 0, qiss1 = 0;  // Q loads issued per slot
    bool ok = true;
    int k = 0;
    bool slot_free = true;  // slot k % kSlots may be written without a wait
    for (;;) {
      unsigned taken = 0;
      if (lane == 0) taken = atomicAdd(&g_sched[sched_slot].next, 1u);
      taken = __shfl_sync(0xffffffffu, taken, 0);
      const bool have = taken < (unsigned)n_items;
      const int item = (int)taken;
      const int slot = k % kSlots;
      if (!slot_free) {
        if (lane == 0)
          ok = mbar_wait(&bars.list_empty[slot], ((k / kSlots) - 1) & 1, &abort_sh, a.status,
                         kWaitLimitNs);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        slot_free = true;
      }
      Slot& S = slots[slot];
      if (!have) {
        if (lane == 0) {
          S.item = -1;
          S.n_ent = 0;
          mbar_arrive(&bars.list_full[slot]);
        }
        break;
      }
      const int b = item / (a.H * n_qt);
      const int h = (item / n_qt) % a.H;
      const int t0 = (item % n_qt) * kBM;
      // kept 64-token key sub-blocks of the two query halves, as bitmaps
      for (int w = lane; w < kMaxSub / 32; w += 32) bmask[0][w] = bmask[1][w] = 0;
      __syncwarp();
      if (a.row_ptr == nullptr) {
        for (int s = lane; s < nsub; s += 32) {
          atomicOr(&bmask[0][s / 32], 1u << (s % 32));
          if (t0 + 64 < a.L) atomicOr(&bmask[1][s / 32], 1u << (s % 32));
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
      // ascending union with per-half keep bits: lane w handles bitmap word w
      const uint32_t w0 = bmask[0][lane], w1 = bmask[1][lane];
      const uint32_t wu = w0 | w1;
      const int c = __popc(wu);
      int incl = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int n_ent = __shfl_sync(0xffffffffu, incl, 31);
      if (n_ent == 0) {
        write_empty_tile<D>(a, b, h, t0, lane);
        __syncwarp();
        continue;  // the slot stays free for the next item
      }
      int pos = incl - c;
      for (uint32_t mb = wu; mb; mb &= mb - 1) {
        const int bit = __ffs(mb) - 1;
        const uint32_t keep = ((w0 >> bit) & 1u) | (((w1 >> bit) & 1u) << 1);
        S.ent[pos++] = (uint32_t)(lane * 32 + bit) | (keep << 16);
      }
      if (lane == 0) {
        S.item = item;
        S.n_ent = n_ent;
        S.b = b;
        S.h = h;
        S.t0 = t0;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.list_full[slot]);
        // Q tile of the item; the slot's previous Q is free once the S
        // products that read it completed
        const int qiss = slot ? qiss1 : qiss0;
        if (qiss > 0)
          ok = mbar_wait(&bars.q_empty[slot], (qiss - 1) & 1, &abort_sh, a.status, kWaitLimitNs);
        if (ok) {
          uint8_t* sq = dsm + Lay::kOffQ + slot * Lay::kQBytes;
          mbar_arrive_expect_tx(&bars.q_full[slot], Lay::kQBytes);
          for (int cc = 0; cc < Lay::kChunks; ++cc)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(sq + cc * Lay::kChunkRowsQ + s * kBox, &tmq, &bars.q_full[slot],
                          cc * 64, t0 + 64 * s, h, b);
          if (slot) ++qiss1; else ++qiss0;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++k;
      slot_free = k < kSlots;
    }
    if (lane == 0) {
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Drain: the Q copies issued above land before the CTA exits.
      volatile int no_abort = 0;
      for (int s = 0; s < kSlots; ++s) {
        const int qiss = s ? qiss1 : qiss0;
        if (qiss > 0 &&
            !mbar_wait(&bars.q_full[s], (qiss - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
      }
    }
  } else if (warp == 0 || warp == kVWarp) {
    // ================================================= K and V producers
    const bool isk = warp == 0;
    uint64_t* full = isk ? bars.kfull : bars.vfull;
    uint64_t* empty = isk ? bars.kempty : bars.vempty;
    const CUtensorMap* tm = isk ? &tmk : &tmv;
    uint8_t* ring = dsm + (isk ? Lay::kOffK : Lay::kOffV);
    const int group = a.H / a.Hkv;
    if (lane == 0) {
      prefetch_tensormap(tm);
      if (isk) prefetch_tensormap(&tmq);
      int g = 0;  // global step: ring stage g % kStages
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kSlots;
        if (!(ok = mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, &abort_sh, a.status,
                             kWaitLimitNs)))
          break;
        const Slot& S = slots[slot];
        if (S.item < 0) break;
        const int n_ent = S.n_ent, b = S.b, kh = S.h / group;
        const int steps = (n_ent + 1) / 2;
        for (int j = 0; j < steps; ++j, ++g) {
          const uint32_t e0 = S.ent[2 * j];
          const uint32_t e1 = (2 * j + 1 < n_ent) ? S.ent[2 * j + 1] : e0;
          const int sub0 = (int)(e0 & 0xFFFFu), sub1 = (int)(e1 & 0xFFFFu);
          const int st = g % kStages;
          if (g >= kStages &&
              !(ok = mbar_wait(&empty[st], ((g / kStages) - 1) & 1, &abort_sh, a.status,
                               kWaitLimitNs)))
            break;
          uint8_t* dst = ring + st * Lay::kKVBytes;
          mbar_arrive_expect_tx(&full[st], Lay::kKVBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, tm, &full[st], c * 64,
                          (s ? sub1 : sub0) * kSubBlock, kh, b);
        }
        if (ok) mbar_arrive(&bars.list_empty[slot]);
      }
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Drain: every copy issued above lands before the CTA exits.
      volatile int no_abort = 0;
      for (int st = (g > kStages ? g - kStages : 0); st < g; ++st)
        if (!mbar_wait(&full[st % kStages], (st / kStages) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kBM, D, true);
      const uint32_t q_base = smem_u32(dsm + Lay::kOffQ);
      const uint32_t k_base = smem_u32(dsm + Lay::kOffK);
      const uint32_t v_base = smem_u32(dsm + Lay::kOffV);
      int quse0 = 0, quse1 = 0;  // Q tiles consumed per slot
      int ouse0 = 0, ouse1 = 0;  // items accumulated per O slot
      bool ok = true;

      // Opens publication ordinal k: its step count, or -1 at the end.
      auto open_item = [&](int k) -> int {
        const int slot = k % kSlots;
        if (!mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, &abort_sh, a.status,
                       kWaitLimitNs)) {
          ok = false;
          return -1;
        }
        const Slot& S = slots[slot];
        if (S.item < 0) return -1;
        if (!mbar_wait(&bars.q_full[slot], (slot ? quse1 : quse0) & 1, &abort_sh, a.status,
                       kWaitLimitNs)) {
          ok = false;
          return -1;
        }
        if (slot) ++quse1; else ++quse0;
        tc_fence_after();
        return (S.n_ent + 1) / 2;
      };
      auto issue_s = [&](int g, int qslot) -> bool {
        const int st = g % kStages;
        if (!mbar_wait(&bars.kfull[st], (g / kStages) & 1, &abort_sh, a.status, kWaitLimitNs))
          return false;
        tc_fence_after();
        const uint32_t kb = k_base + st * Lay::kKVBytes;
        const uint32_t qb = q_base + qslot * Lay::kQBytes;
        const uint32_t dcol = tmem + kColS + 128u * (uint32_t)(g & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk % 4) * 32;  // 16 bf16 of K inside the swizzle atom
          const uint64_t ad = smem_desc_sw128(qb + (kk / 4) * Lay::kChunkRowsQ + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kb + (kk / 4) * Lay::kChunkRowsKV + off, 16, 1024);
          mma_bf16_ss(dcol, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars.kempty[st]);
        tc_commit(&bars.s[g & 1]);
        return true;
      };

      int k = 0, j = 0, g = 0;
      int steps = open_item(0);
      if (steps > 0) {
        ok = issue_s(0, 0);
        if (ok && steps == 1) tc_commit(&bars.q_empty[0]);
      }
      while (ok && steps > 0) {
        // S of the next step, into the next item when this one ends here
        int k2 = k, j2 = j + 1, steps2 = steps;
        if (j2 == steps) {
          k2 = k + 1;
          j2 = 0;
          steps2 = open_item(k2);
          if (!ok) break;
        }
        if (steps2 > 0) {
          if (!(ok = issue_s(g + 1, k2 % kSlots))) break;
          if (j2 == steps2 - 1) tc_commit(&bars.q_empty[k2 % kSlots]);
        }
        // O += P V for the current step
        const int slot = k % kSlots;
        if (!(ok = mbar_wait(&bars.p[g & 1], (g >> 1) & 1, &abort_sh, a.status, kWaitLimitNs)))
          break;
        const int st = g % kStages;
        if (!(ok = mbar_wait(&bars.vfull[st], (g / kStages) & 1, &abort_sh, a.status,
                             kWaitLimitNs)))
          break;
        const int ouse = slot ? ouse1 : ouse0;
        if (j == 0 && ouse > 0 &&
            !(ok = mbar_wait(&bars.o_empty[slot], (ouse - 1) & 1, &abort_sh, a.status,
                             kWaitLimitNs)))
          break;
        tc_fence_after();
        const uint32_t vb = v_base + st * Lay::kKVBytes;
        const uint32_t pcol = tmem + kColS + 128u * (uint32_t)(g & 1);
        const uint32_t ocol = tmem + kColO + 128u * (uint32_t)slot;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(vb + kk * 16 * 128, Lay::kChunkRowsKV, 1024);
          // P elements [16 kk, 16 kk + 16): columns 64 (kk / 4) + 8 (kk % 4)
          mma_bf16_ts(ocol, pcol + 64 * (kk / 4) + 8 * (kk % 4), bd, idPV,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars.vempty[st]);
        tc_commit(&bars.o);
        if (j == steps - 1) {
          tc_commit(&bars.o_full[slot]);
          if (slot) ++ouse1; else ++ouse0;
          mbar_arrive(&bars.list_empty[slot]);
        }
        k = k2;
        j = j2;
        steps = steps2;
        ++g;
      }
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Every MMA issued above completes before TMEM is released.
      tc_commit(&bars.done);
      volatile int no_abort = 0;
      if (!mbar_wait(&bars.done, 0, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
    }
  } else {
    // ============================================================ softmax
    // Two warpgroups: group g owns key columns [64 g, 64 g + 64) of each S
    // row (key sub-block g of the step) and columns [d/2 g, d/2 g + d/2) of
    // O.  The two threads of a row swap their tile maxima through shared
    // memory once per step.  Each group writes its half of P (bf16 pairs)
    // over the first 32 of its own 64 S columns, so neither group overwrites
    // S the other may still read.
    const int grp = (warp - 2) / 4;
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = a.scale_log2;
    uint32_t soft_uses = 0;
    int ouse0 = 0, ouse1 = 0;  // items finished per O slot
    int g = 0;  // global step
    bool ok = true;
    for (int k = 0;; ++k) {
      const int slot = k % kSlots;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, &abort_sh,
                                             a.status, kWaitLimitNs));
      if (!ok) break;
      const Slot& S = slots[slot];
      if (S.item < 0) break;
      const int n_ent = S.n_ent, b = S.b, h = S.h, t = S.t0 + row;
      const int n_steps = (n_ent + 1) / 2;
      float m = -INFINITY;  // running max (log2 units) used as the exponent reference
      float l = 0.f;        // this half-row's sum of the bf16-rounded weights
      float lx = 0.f;       // this half-row's sum of the unrounded weights (LSE only)
      const uint32_t ocol = trow + kColO + 128u * (uint32_t)slot + (D / 2) * grp;
      for (int j = 0; j < n_steps; ++j, ++g) {
        const int buf = g & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.s[buf], (g >> 1) & 1, &abort_sh, a.status,
                                               kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t e0 = S.ent[2 * j];
        const uint32_t e1 = (2 * j + 1 < n_ent) ? S.ent[2 * j + 1] : (e0 & 0xFFFFu);
        // (keep is uniform over a warp: its 32 rows lie in one query block)
        const bool keep = ((grp ? e1 : e0) >> (16 + half)) & 1u;
        const uint32_t scol = trow + kColS + 128u * (uint32_t)buf + 64 * grp;
        float sv[64];
        {
          uint32_t r[64];
          tmem_ld32(scol, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 64; ++x) sv[x] = keep ? __uint_as_float(r[x]) * sl2 : -INFINITY;
        }
        float mt = -INFINITY;
#pragma unroll
        for (int x = 0; x < 64; x += 2) mt = fmaxf(mt, fmaxf(sv[x], sv[x + 1]));
        sh_max[buf][grp][row] = mt;
        if (!(ok = group_sync(&bars.soft, soft_uses, &abort_sh, a.status, kWaitLimitNs))) break;
        mt = fmaxf(mt, sh_max[buf][grp ^ 1][row]);
        const bool raise = mt > m + 8.0f;
        if (__any_sync(0xffffffffu, raise)) {
          if (j > 0) {
            // O must hold every product of this item issued so far before it
            // is rescaled.  PV(g-2) is complete (S(g) was committed after it)
            // and PV(g) cannot start before this step's P, so the parity of
            // PV(g-1) names one completion.
            ok = __all_sync(0xffffffffu, mbar_wait(&bars.o, (g - 1) & 1, &abort_sh, a.status,
                                                   kWaitLimitNs));
            if (!ok) break;
            tc_fence_after();
            const float alpha = raise ? ex2_approx(m - mt) : 1.0f;
            l *= alpha;
            lx *= alpha;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              uint32_t ov[32];
              tmem_ld32(ocol + c * 32, ov);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
              tmem_st32(ocol + c * 32, ov);
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
        // bf16 pairs of P over this half's own S columns; l sums the rounded weights
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
        tmem_st32(scol, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p[buf]);
      }
      if (!ok) break;
      // --------------------------------------------------------- epilogue
      sh_sum[0][grp][row] = l;
      sh_sum[1][grp][row] = lx;
      if (!(ok = group_sync(&bars.soft, soft_uses, &abort_sh, a.status, kWaitLimitNs))) break;
      l += sh_sum[0][grp ^ 1][row];
      lx += sh_sum[1][grp ^ 1][row];
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.o_full[slot], (slot ? ouse1 : ouse0) & 1,
                                             &abort_sh, a.status, kWaitLimitNs));
      if (!ok) break;
      if (slot) ++ouse1; else ++ouse0;
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                          (int64_t)t * a.os[1] + h * a.os[2] + (D / 2) * grp;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[32];
        tmem_ld32(ocol + c * 32, ov);
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.o_empty[slot]);
        mbar_arrive(&bars.list_empty[slot]);
      }
      if (a.lse && grp == 0 && t < a.L)
        a.lse[((int64_t)b * a.H + h) * a.L + t] =
            lx > 0.f ? (m + log2f(lx)) * 0.69314718055994531f : -INFINITY;
    }
    if (!ok) raise_timeout(&abort_sh, a.status);
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    // this CTA takes no more items; the last one out resets the counter
    __threadfence();
    if (atomicAdd(&g_sched[sched_slot].finished, 1u) == gridDim.x - 1) {
      atomicExch(&g_sched[sched_slot].next, 0u);
      atomicExch(&g_sched[sched_slot].finished, 0u);
    }
  }
}

int g_num_sms[64] = {0};
std::atomic<unsigned> g_launches{0};

template <int D, bool kLse>
cudaError_t launch_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                      const CUtensorMap* tv, cudaStream_t st, int grid) {
  using Lay = Layout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, kLse>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
  if (e != cudaSuccess) return e;
  const int slot = (int)(g_launches.fetch_add(1u) % kSchedRing);
  attn_tc_kernel<D, kLse><<<grid, kThreads, Lay::kSmem, st>>>(*tq, *tk, *tv, a, slot);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_num_sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  // one persistent CTA per SM (the shared-memory footprint admits one)
  const int64_t n_items = (int64_t)a.B * a.H * ((a.L + kBM - 1) / kBM);
  const int grid = (int)(n_items < g_num_sms[dev] ? n_items : g_num_sms[dev]);
  if (a.d == 128)
    return a.lse ? launch_tc<128, true>(a, tq, tk, tv, st, grid)
                 : launch_tc<128, false>(a, tq, tk, tv, st, grid);
  return a.lse ? launch_tc<64, true>(a, tq, tk, tv, st, grid)
               : launch_tc<64, false>(a, tq, tk, tv, st, grid);
}

}  // namespace sdl
