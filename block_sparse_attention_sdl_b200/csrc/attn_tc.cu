// bf16 block-sparse / dense attention on sm_100a tensor cores.
//
// The fused IO-aware block-sparse kernel of the Step-dLLM abstract,
// re-designed for Blackwell.  A work item is a 128-row query tile of one
// head; it walks the kept key blocks of its rows, two 64-token sub-blocks
// (128 keys) per step.  CTAs are persistent and small enough that two run
// on every SM; each works through one item at a time, so the two CTAs of an
// SM interleave on its tensor cores (one's softmax overlaps the other's
// products) without waiting on each other.  Items come from a global
// counter, first come first served (tiles differ in cost by the length of
// their kept lists).
//
//   warp 0        loads: takes items and copies an item's prebuilt list
//                 (tile_lists_kernel, run once per mask) or builds the union
//                 list of its two query blocks into a list slot (three slots,
//                 the next item's list while the current item runs); per item
//                 its Q tile, per step its K and V sub-blocks by TMA
//                 (128-byte-swizzled 64x64 boxes) into one K and one V stage.
//                 Items whose lists are empty (only a caller's mask can have
//                 empty rows) are written here as zero rows.
//   warp 1        TMEM allocator and MMA issuer (one thread):
//                   S = Q K^T    tcgen05.mma kind::f16, A and B from shared
//                                memory, M=128, N=128, fp32 in TMEM;
//                   O += P V     A = P (bf16, over S's first 64 TMEM
//                                columns), B = V from shared memory
//                                (N-major), M=128, N=d; issued in two
//                                halves, keys 0..63 as soon as the softmax
//                                has written their weights.
//                 The next S is issued after the PV product (the two share
//                 S's columns), which also leaves O quiescent for the
//                 softmax once that S product has completed.
//   warps 2-5     softmax: one thread per query row (its TMEM lane), all 128
//                 columns of the step.  Online softmax in the log2 domain;
//                 the running max is raised only when it grows by more than
//                 8 (a factor 256), and O is rescaled in TMEM only then; P
//                 written back as bf16, the row sum taken over those rounded
//                 weights (the LSE's over the fp32 weights).  Epilogue per
//                 item: O / l rounded to bf16 and written by TMA tensor
//                 stores from a per-warp shared-memory box, LSE.
//
// With 64-token blocks a 128-row tile covers two query blocks; the item walks
// the union of their kept lists and masks, per 64x64 quadrant, the key
// sub-blocks a query block did not keep.  With 128-token blocks both halves
// share one list.  Dense attention is the same walk over every sub-block.
//
// TMEM (256 columns per CTA): S at column 0, O at 128.
// Every mbarrier wait is bounded; on timeout the CTA raises the device status
// word, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "internal.cuh"
#include "ptx.cuh"

namespace sdl {
namespace {

constexpr int kBM = 128;         // query rows per item
constexpr int kBN = 128;         // key rows per step
constexpr int kSlots = 3;        // list slots
constexpr int kMaxSub = 1024;    // 64-token sub-blocks per sequence (L <= 65536)
constexpr int kThreads = 192;    // 6 warps
constexpr int kCtasPerSm = 2;
constexpr int kLoadWarp = 0, kMmaWarp = 1, kSoftWarp0 = 2;
constexpr int kBox = 64 * 128;   // bytes of one 64-row x 64-column bf16 box
constexpr int kOBoxBytes = 32 * 64;  // one 32-row x 32-column bf16 output box
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 128;
// PV issued in two halves, the first once the softmax has written keys 0..63
constexpr bool kSplitPV = true;

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;           // 128-byte column chunks
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;     // one stage of K (or V)
  static constexpr int kChunkRowsQ = kBM * 128;    // bytes per Q column chunk
  static constexpr int kChunkRowsKV = kBN * 128;   // bytes per K/V column chunk
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKVBytes;
  // output staging: per softmax warp one 32-row x 32-column bf16 box
  // (64-byte rows, 64-byte swizzle) for the tensor stores of O
  static constexpr int kOffO = kOffV + kKVBytes;
  static constexpr int kBytes = kOffO + 4 * kOBoxBytes;
  static constexpr int kSmem = kBytes + 1024;      // + alignment slack
};
// two CTAs per SM: 228 KB of shared memory per SM, 1 KB of it reserved per
// CTA, and up to 8 KB of static shared memory per CTA
static_assert(kCtasPerSm * (Layout<128>::kSmem + 8192 + 1024) <= 228 * 1024, "shared memory");

// Consumers of a list slot: the MMA warp and the 4 softmax warps.
constexpr int kListConsumers = 1 + 4;

struct Bars {
  uint64_t list_full[kSlots];   // slot published by the load warp
  uint64_t list_empty[kSlots];  // slot released by every consumer
  uint64_t q_full, q_empty;     // Q landed / the item's S products completed
  uint64_t kfull, kempty, vfull, vempty;
  uint64_t s_full;              // S written
  uint64_t p_half;              // P of keys 0..63 written (one arrival per softmax warp)
  uint64_t p_full;              // all of P written (one arrival per softmax warp)
  uint64_t o_full;              // every product of the item completed
  uint64_t done;
};

// One published item: its kept list, entries sub-block index | keep bits << 14
// (bit 14: query rows 0..63 keep it, bit 15: rows 64..127).
struct Slot {
  int item;  // -1: end of the CTA's items
  int n_ent;
  int b, h;
  int t0, t1;  // first tokens of the tile's two 64-row halves (L: half unused)
  uint16_t ent[kMaxSub];
};
constexpr uint32_t kKeepShift = 14;
constexpr uint32_t kSubMask = (1u << kKeepShift) - 1u;

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
__device__ __forceinline__ void write_empty_tile(const AttnArgs& a, int b, int h, int t0, int t1,
                                                 int lane) {
  for (int r = lane; r < kBM; r += 32) {
    const int t = (r < 64 ? t0 : t1) + (r & 63);
    if (t >= a.L) continue;
    uint4* op = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                                         (int64_t)t * a.os[1] + h * a.os[2]);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) op[c] = make_uint4(0, 0, 0, 0);
    if (a.lse) a.lse[((int64_t)b * a.H + h) * a.L + t] = -INFINITY;
  }
}

// The tile of `item`: batch element, head and first tokens of its two 64-row
// halves (L: half unused), from the plan for 64-token blocks, else adjacent.
__device__ __forceinline__ void tile_of(const AttnArgs& a, int item, int n_qt, int& b, int& h,
                                        int& t0, int& t1) {
  b = item / (a.H * n_qt);
  h = (item / n_qt) % a.H;
  if (a.plan != nullptr) {
    // the tile's two query blocks from the plan (64-token blocks)
    const int qb0 = a.plan[2 * (int64_t)item], qb1 = a.plan[2 * (int64_t)item + 1];
    if (qb0 >= a.nb || qb0 < -1 || qb1 >= a.nb || qb1 < -1) atomicOr(a.status, kDevBadMask);
    t0 = (qb0 >= 0 && qb0 < a.nb) ? qb0 * 64 : a.L;
    t1 = (qb1 >= 0 && qb1 < a.nb) ? qb1 * 64 : a.L;
  } else {
    t0 = (item % n_qt) * kBM;
    t1 = t0 + 64 < a.L ? t0 + 64 : a.L;
  }
}

// The kept 64-token key sub-blocks of a tile's two query halves, as bitmaps
// in `bmask` (all key sub-blocks without a mask), listed in ascending order
// with their keep bits into `ent` (shared or global memory); all lanes of one
// warp.  Returns the list's length.
__device__ int union_list(const AttnArgs& a, int b, int h, int t0, int t1,
                          uint32_t (*bmask)[kMaxSub / 32], uint16_t* ent, int lane) {
  const int nsub = a.Lk / kSubBlock;
  for (int w = lane; w < kMaxSub / 32; w += 32) bmask[0][w] = bmask[1][w] = 0;
  __syncwarp();
  if (a.row_ptr == nullptr) {
    for (int s = lane; s < nsub; s += 32) {
      if (t0 < a.L) atomicOr(&bmask[0][s / 32], 1u << (s % 32));
      if (t1 < a.L) atomicOr(&bmask[1][s / 32], 1u << (s % 32));
    }
  } else {
    const int per = a.block / kSubBlock;  // sub-blocks per block: 1 or 2
    const int rows_in_tile = a.block == 64 ? 2 : 1;
    for (int rr = 0; rr < rows_in_tile; ++rr) {
      const int tr = rr ? t1 : t0;
      if (tr >= a.L) continue;
      const int i = tr / a.block;
      const int64_t r = ((int64_t)b * a.H + h) * a.nb + i;
      const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
      for (int x = beg + lane; x < end; x += 32) {
        const int jb = a.col_idx[x];
        const bool bad_range = jb < 0 || jb >= a.nb;
        if (bad_range || (x > beg && a.col_idx[x - 1] >= jb)) atomicOr(a.status, kDevBadMask);
        if (bad_range) continue;
        for (int u = 0; u < per; ++u) {
          const int s = jb * per + u;
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
  int pos = incl - c;
  for (uint32_t mb = wu; mb; mb &= mb - 1) {
    const int bit = __ffs(mb) - 1;
    const uint32_t keep = ((w0 >> bit) & 1u) | (((w1 >> bit) & 1u) << 1);
    ent[pos++] = (uint16_t)((uint32_t)(lane * 32 + bit) | (keep << kKeepShift));
  }
  __syncwarp();
  return n_ent;
}

// Prebuilt tile lists (sdl_tile_lists): per position r of the take order a
// record of 8 int32 {item, n_ent, t0, t1, 0, 0, 0, 0}, then per position
// `cap` 16-bit entries (the union list, as in a list slot).
constexpr int kListRecInts = 8;
__host__ __device__ inline int lists_cap(int Lk) { return ((Lk / kSubBlock) + 7) / 8 * 8; }
__host__ __device__ inline size_t lists_bytes(int64_t n_items, int Lk) {
  return (size_t)n_items * (kListRecInts * 4 + 2 * (size_t)lists_cap(Lk));
}

// Takes items until a non-empty one and writes its union list into S (all
// lanes of one warp; lane 0 writes the header).  Returns false once the
// launch's items are used up (S then holds the end marker).  With prebuilt
// lists the r-th item taken is record r, copied; else the r-th is order[r]
// (or r) and its list is built here.
template <int D>
__device__ bool build_item(const AttnArgs& a, const CUtensorMap* tmq, Slot& S,
                           uint32_t (*bmask)[kMaxSub / 32], int sched_slot, int n_items, int n_qt,
                           int lane) {
  const int nsub = a.Lk / kSubBlock;
  for (;;) {
    unsigned taken = 0;
    if (lane == 0) taken = atomicAdd(&g_sched[sched_slot].next, 1u);
    taken = __shfl_sync(0xffffffffu, taken, 0);
    if (taken >= (unsigned)n_items) break;
    int item = (int)taken, n_ent = 0, b, h, t0, t1;
    if (a.lists != nullptr) {
      const int4 rec = *reinterpret_cast<const int4*>(a.lists + (int64_t)taken * kListRecInts);
      item = rec.x;
      n_ent = rec.y;
      if (item < 0 || item >= n_items || n_ent < 0 || n_ent > nsub) {
        if (lane == 0) atomicOr(a.status, kDevBadMask);
        continue;
      }
      b = item / (a.H * n_qt);
      h = (item / n_qt) % a.H;
      t0 = rec.z;
      t1 = rec.w;
      if (t0 < 0 || t0 > a.L || t1 < 0 || t1 > a.L) {
        if (lane == 0) atomicOr(a.status, kDevBadMask);
        continue;
      }
      const uint16_t* src = reinterpret_cast<const uint16_t*>(a.lists + (int64_t)n_items *
                                                                            kListRecInts) +
                            (int64_t)taken * lists_cap(a.Lk);
      for (int x = lane; x < n_ent; x += 32) {
        uint16_t e = src[x];
        if ((int)(e & kSubMask) >= nsub) {
          atomicOr(a.status, kDevBadMask);
          e = 0;
        }
        S.ent[x] = e;
      }
      __syncwarp();
    } else {
      if (a.order != nullptr) {
        // costliest tiles first (the order is a permutation of the items)
        const int o = a.order[item];
        if (o < 0 || o >= n_items) {
          if (lane == 0) atomicOr(a.status, kDevBadMask);
          continue;
        }
        item = o;
      }
      tile_of(a, item, n_qt, b, h, t0, t1);
      n_ent = union_list(a, b, h, t0, t1, bmask, S.ent, lane);
    }
    if (n_ent == 0) {
      write_empty_tile<D>(a, b, h, t0, t1, lane);
      __syncwarp();
      continue;
    }
    if (lane == 0) {
      S.item = item;
      S.n_ent = n_ent;
      S.b = b;
      S.h = h;
      S.t0 = t0;
      S.t1 = t1;
      // its Q tile is loaded when the current item's S products are done; warm L2 now
      for (int cc = 0; cc < D / 64; ++cc)
        for (int s = 0; s < 2; ++s)
          if ((s ? t1 : t0) < a.L) tma_prefetch_l2_4d(tmq, cc * 64, s ? t1 : t0, h, b);
    }
    __syncwarp();
    return true;
  }
  if (lane == 0) {
    S.item = -1;
    S.n_ent = 0;
  }
  __syncwarp();
  return false;
}

// One warp per position r of the take order: record r of the prebuilt lists
// (the tile order[r], or r, and its union list).
constexpr int kListWarps = 8;
__global__ void __launch_bounds__(kListWarps * 32) tile_lists_kernel(AttnArgs a, int32_t* lists) {
  __shared__ uint32_t bm[kListWarps][2][kMaxSub / 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = (a.L + kBM - 1) / kBM;
  const int n_items = a.B * a.H * n_qt;
  const int r = blockIdx.x * kListWarps + warp;
  if (r >= n_items) return;
  int item = r;
  if (a.order != nullptr) {
    item = a.order[r];
    if (item < 0 || item >= n_items) {
      if (lane == 0) {
        atomicOr(a.status, kDevBadMask);
        *reinterpret_cast<int4*>(lists + (int64_t)r * kListRecInts) = make_int4(-1, 0, 0, 0);
      }
      return;
    }
  }
  int b, h, t0, t1;
  tile_of(a, item, n_qt, b, h, t0, t1);
  uint16_t* ent = reinterpret_cast<uint16_t*>(lists + (int64_t)n_items * kListRecInts) +
                  (int64_t)r * lists_cap(a.Lk);
  const int n_ent = union_list(a, b, h, t0, t1, bm[warp], ent, lane);
  if (lane == 0) {
    int4* rec = reinterpret_cast<int4*>(lists + (int64_t)r * kListRecInts);
    rec[0] = make_int4(item, n_ent, t0, t1);
    rec[1] = make_int4(0, 0, 0, 0);
  }
}

template <int D, bool kLse>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                   AttnArgs a, int sched_slot) {
  using Lay = Layout<D>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                            ~(uintptr_t)1023);
  __shared__ Bars bars;
  __shared__ Slot slots[kSlots];
  __shared__ uint32_t bmask[2][kMaxSub / 32];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = (a.L + kBM - 1) / kBM;
  const int n_items = a.B * a.H * n_qt;

  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int s = 0; s < kSlots; ++s) {
        mbar_init(&bars.list_full[s], 1);
        mbar_init(&bars.list_empty[s], kListConsumers);
      }
      mbar_init(&bars.q_full, 1);
      mbar_init(&bars.q_empty, 1);
      mbar_init(&bars.kfull, 1);
      mbar_init(&bars.kempty, 1);
      mbar_init(&bars.vfull, 1);
      mbar_init(&bars.vempty, 1);
      mbar_init(&bars.s_full, 1);
      mbar_init(&bars.p_half, 4);
      mbar_init(&bars.p_full, 4);
      mbar_init(&bars.o_full, 1);
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
  // (The load and MMA roles run warp-converged; one elected lane issues their
  // copies, MMAs and arrivals, and every wait is made warp-uniform.)

  if (warp == kLoadWarp) {
    // ================================================================ loads
    const bool leader = elect_one_sync();
    if (leader) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
    const int group = a.H / a.Hkv;
    bool ok = true;
    int built = 0;   // lists published (the end marker included)
    bool ended = false;
    int nq = 0;      // Q tiles loaded
    int g = 0;       // steps loaded (K and V stage phases)
    int gk = 0, gv = 0;  // K and V copies issued (one ahead of g between a step's copies)
    // publishes the next list into its slot once the slot's item is done
    auto publish_next = [&]() -> bool {
      const int slot = built % kSlots;
      if (built >= kSlots &&
          !__all_sync(0xffffffffu, mbar_wait(&bars.list_empty[slot], ((built / kSlots) - 1) & 1,
                                             &abort_sh, a.status, kWaitLimitNs)))
        return false;
      ended = !build_item<D>(a, &tmq, slots[slot], bmask, sched_slot, n_items, n_qt, lane);
      if (lane == 0) mbar_arrive(&bars.list_full[slot]);
      ++built;
      return true;
    };
    ok = publish_next();
    for (int k = 0; ok; ++k) {
      const Slot& S = slots[k % kSlots];
      if (S.item < 0) break;
      const int n_ent = S.n_ent, kh = S.h / group, b = S.b;
      // Q of the item, once the previous item's S products have completed
      if (nq > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&bars.q_empty, (nq - 1) & 1,
                                                             &abort_sh, a.status, kWaitLimitNs))))
        break;
      if (leader) {
        uint8_t* sq = dsm + Lay::kOffQ;
        mbar_arrive_expect_tx(&bars.q_full, Lay::kQBytes);
        for (int cc = 0; cc < Lay::kChunks; ++cc)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(sq + cc * Lay::kChunkRowsQ + s * kBox, &tmq, &bars.q_full, cc * 64,
                        s ? S.t1 : S.t0, S.h, b);
      }
      ++nq;
      const int n_steps = (n_ent + 1) / 2;
      for (int j = 0; j < n_steps; ++j, ++g) {
        const uint32_t e0 = S.ent[2 * j];
        const uint32_t e1 = (2 * j + 1 < n_ent) ? S.ent[2 * j + 1] : e0;
        const int sub0 = (int)(e0 & kSubMask), sub1 = (int)(e1 & kSubMask);
        // K of the step once the previous S product has completed
        if (g > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&bars.kempty, (g - 1) & 1,
                                                              &abort_sh, a.status, kWaitLimitNs))))
          break;
        if (leader) {
          uint8_t* dst = dsm + Lay::kOffK;
          mbar_arrive_expect_tx(&bars.kfull, Lay::kKVBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, &tmk, &bars.kfull, c * 64,
                          (s ? sub1 : sub0) * kSubBlock, kh, b);
        }
        gk = g + 1;
        // the next item's list, while this one runs
        if (j == 0 && !ended && !(ok = publish_next())) break;
        // V of the step once the previous PV product has completed
        if (g > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&bars.vempty, (g - 1) & 1,
                                                              &abort_sh, a.status, kWaitLimitNs))))
          break;
        if (leader) {
          uint8_t* dst = dsm + Lay::kOffV;
          mbar_arrive_expect_tx(&bars.vfull, Lay::kKVBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, &tmv, &bars.vfull, c * 64,
                          (s ? sub1 : sub0) * kSubBlock, kh, b);
        }
        gv = g + 1;
      }
    }
    if (leader) {
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Drain: every copy issued above lands before the CTA exits.  The K and V
      // copies are counted apart: a step left early has its K copy in flight.
      volatile int no_abort = 0;
      if (gk > 0 && !mbar_wait(&bars.kfull, (gk - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
      if (gv > 0 && !mbar_wait(&bars.vfull, (gv - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
      if (nq > 0 && !mbar_wait(&bars.q_full, (nq - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA
    const bool leader = elect_one_sync();
    constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, false);
    constexpr uint32_t idPV = idesc_bf16_f32(kBM, D, true);
    // Descriptors are built once: the start-address field (bits 0..13,
    // address >> 4) of the descriptor for address x + off is the base
    // descriptor's plus off >> 4, without carry (shared addresses < 2^18).
    const uint64_t dq = smem_desc_sw128(smem_u32(dsm + Lay::kOffQ), 16, 1024);
    const uint64_t dk = smem_desc_sw128(smem_u32(dsm + Lay::kOffK), 16, 1024);
    const uint64_t dv = smem_desc_sw128(smem_u32(dsm + Lay::kOffV), Lay::kChunkRowsKV, 1024);
    const uint32_t scol = tmem + kColS, ocol = tmem + kColO;
    bool ok = true;
    int n = 0;  // steps issued
    for (int k = 0; ok; ++k) {
      const int slot = k % kSlots;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.list_full[slot], (k / kSlots) & 1,
                                                   &abort_sh, a.status, kWaitLimitNs))))
        break;
      const Slot& S = slots[slot];
      if (S.item < 0) break;
      const int n_steps = (S.n_ent + 1) / 2;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.q_full, k & 1, &abort_sh, a.status,
                                                   kWaitLimitNs))))
        break;
      for (int j = 0; j < n_steps; ++j, ++n) {
        const bool last = j == n_steps - 1;
        // S = Q K^T (the previous PV product, which reads S's columns, was issued before)
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.kfull, n & 1, &abort_sh, a.status,
                                                     kWaitLimitNs))))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 d-columns: chunk kk / 4, 32 bytes (kk % 4) inside the swizzle atom
          const uint64_t offq = (uint64_t)(((kk / 4) * Lay::kChunkRowsQ + (kk % 4) * 32) >> 4);
          const uint64_t offk = (uint64_t)(((kk / 4) * Lay::kChunkRowsKV + (kk % 4) * 32) >> 4);
          if (leader) mma_bf16_ss(scol, dq + offq, dk + offk, idS, kk > 0 ? 1u : 0u);
        }
        if (leader) {
          tc_commit(&bars.kempty);
          tc_commit(&bars.s_full);
          if (last) tc_commit(&bars.q_empty);
        }
        // O += P V in two halves: keys 0..63 once the softmax has written their
        // weights (the product runs while it computes the rest), then keys 64..127
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(kSplitPV ? &bars.p_half : &bars.p_full, n & 1,
                                                     &abort_sh, a.status, kWaitLimitNs))))
          break;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.vfull, n & 1, &abort_sh, a.status,
                                                     kWaitLimitNs))))
          break;
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {
          if (kSplitPV && hk == 1 &&
              !(ok = __all_sync(0xffffffffu, mbar_wait(&bars.p_full, n & 1, &abort_sh, a.status,
                                                       kWaitLimitNs))))
            break;
          tc_fence_after();
#pragma unroll
          for (int kq = 0; kq < kBN / 32; ++kq) {
            // keys [16 kk, 16 kk + 16): V rows 16 kk.. (128 bytes each); P elements
            // packed in columns [8 kk, 8 kk + 8)
            const int kk = hk * (kBN / 32) + kq;
            if (leader)
              mma_bf16_ts(ocol, scol + 8 * kk, dv + (uint64_t)((kk * 16 * 128) >> 4), idPV,
                          (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (!ok) break;
        if (leader) {
          tc_commit(&bars.vempty);
          if (last) tc_commit(&bars.o_full);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.list_empty[slot]);
    }
    if (leader) {
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Every MMA issued above completes before TMEM is released.
      tc_commit(&bars.done);
      volatile int no_abort = 0;
      if (!mbar_wait(&bars.done, 0, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t scol = trow + kColS;
    const uint32_t ocol = trow + kColO;
    uint8_t* ostage = dsm + Lay::kOffO + (warp - kSoftWarp0) * kOBoxBytes;
    const float sl2 = a.scale_log2;
    int n = 0;  // steps so far
    bool ok = true;
    for (int k = 0;; ++k) {
      const int slot = k % kSlots;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, &abort_sh,
                                             a.status, kWaitLimitNs));
      if (!ok) break;
      const Slot& S = slots[slot];
      if (S.item < 0) break;
      const int n_ent = S.n_ent, b = S.b, h = S.h, tok = (half ? S.t1 : S.t0) + (row & 63);
      const int n_steps = (n_ent + 1) / 2;
      float m = -INFINITY;  // running max (log2 units) used as the exponent reference
      float l = 0.f;        // row sum of the bf16-rounded weights
      float lx = 0.f;       // row sum of the unrounded weights (LSE only)
      for (int j = 0; j < n_steps; ++j, ++n) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars.s_full, n & 1, &abort_sh, a.status, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t e0 = S.ent[2 * j];
        const uint32_t e1 = (2 * j + 1 < n_ent) ? S.ent[2 * j + 1] : (e0 & kSubMask);
        // (keep is uniform over a warp: its 32 rows lie in one query block)
        const bool keep0 = (e0 >> (kKeepShift + half)) & 1u;
        const bool keep1 = (e1 >> (kKeepShift + half)) & 1u;
        uint32_t r[128];
        tmem_ld32(scol + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld32(scol + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
        tmem_ld32(scol + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
        tmem_wait_ld();
        // tile maxima of the two 64-column halves (three-input max)
        float mh[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int x0 = 64 * hf;
          float m0 = __uint_as_float(r[x0]), m1 = __uint_as_float(r[x0 + 1]);
#pragma unroll
          for (int x = x0 + 2; x < x0 + 62; x += 4) {
            m0 = max3f(m0, __uint_as_float(r[x]), __uint_as_float(r[x + 1]));
            m1 = max3f(m1, __uint_as_float(r[x + 2]), __uint_as_float(r[x + 3]));
          }
          mh[hf] = max3f(m0, m1, fmaxf(__uint_as_float(r[x0 + 62]), __uint_as_float(r[x0 + 63])));
        }
        const float mt = fmaxf(keep0 ? mh[0] : -INFINITY, keep1 ? mh[1] : -INFINITY) * sl2;
        const bool raise = mt > m + 8.0f;
        if (__any_sync(0xffffffffu, raise)) {
          if (j > 0) {
            // O is quiescent: this step's S product was issued after the
            // previous PV product and has completed.
            const float alpha = raise ? ex2_approx(m - mt) : 1.0f;
            l *= alpha;
            lx *= alpha;
#pragma unroll 1
            for (int c = 0; c < D / 16; ++c) {
              uint32_t ov[16];
              tmem_ld16(ocol + c * 16, ov);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 16; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
              tmem_st16(ocol + c * 16, ov);
            }
            tmem_wait_st();
          }
          if (raise) m = mt;
        }
        // P = exp2(S * scale * log2e - m) on a kept half, 0 otherwise (a kept
        // half always has a finite reference here: its own maximum raised it);
        // bf16 pairs over S's first 64 columns; l sums the rounded weights, each
        // bf16 half added to an fp32 sum by one mixed-precision add (x = s *
        // scale_log2 - m packed in pairs)
        const uint64_t sl2x2 = pack2(sl2, sl2), nmx2 = pack2(-m, -m);
        float rsa = 0.f, rsb = 0.f;  // row sums of the rounded weights (low, high halves)
        uint64_t rx2 = pack2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 32 weights -> 16 packed columns at a time
          const bool kp = c < 2 ? keep0 : keep1;
          uint32_t pw[16];
          if (kp) {
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const float2 xv = unpack2(fma2(
                  pack2(__uint_as_float(r[32 * c + x]), __uint_as_float(r[32 * c + x + 1])), sl2x2,
                  nmx2));
              const float p0 = ex2_approx(xv.x), p1 = ex2_approx(xv.y);
              __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
              const uint32_t u = *reinterpret_cast<uint32_t*>(&pk);
              asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
                  "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
                  : "+f"(rsa), "+f"(rsb) : "r"(u));
              if constexpr (kLse) rx2 = add2(rx2, pack2(p0, p1));
              pw[x / 2] = u;
            }
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) pw[x] = 0u;
          }
          tmem_st16(scol + 16 * c, pw);
          if (kSplitPV && c == 1) {
            // keys 0..63 are ready for their half of the PV product
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.p_half);
          }
        }
        {
          const float2 b2 = unpack2(rx2);
          l += rsa + rsb;
          lx += b2.x + b2.y;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full);
      }
      if (!ok) break;
      // --------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bars.o_full, k & 1, &abort_sh, a.status, kWaitLimitNs));
      if (!ok) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      // O / l as bf16, 32 columns at a time through this warp's staging box
      // (row `lane` holds its 64 bytes as four 16-byte chunks, chunk x at
      // x ^ ((lane / 2) % 4): the 64-byte swizzle), then one tensor store per
      // box; rows past L are clipped by the store
      const int tok0 = tok - lane;  // first token of this warp's 32 rows
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(ocol + c * 32, ov);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(ov[2 * x]) * inv,
                                                   __uint_as_float(ov[2 * x + 1]) * inv);
          pk[x] = *reinterpret_cast<uint32_t*>(&v);
        }
        if (lane == 0) bulk_wait_read_all();  // the previous box has been read out
        __syncwarp();
        uint4* row_sm = reinterpret_cast<uint4*>(ostage + lane * 64);
#pragma unroll
        for (int x = 0; x < 4; ++x)
          row_sm[x ^ ((lane >> 1) & 3)] =
              make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && tok0 < a.L) {
          tma_store_4d(&tmo, ostage, c * 32, tok0, h, b);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.list_empty[slot]);
      if (a.lse && tok < a.L)
        a.lse[((int64_t)b * a.H + h) * a.L + tok] =
            lx > 0.f ? (m + log2f(lx)) * 0.69314718055994531f : -INFINITY;
    }
    if (lane == 0) bulk_wait_all();  // this warp's output stores have completed
    __syncwarp();
    if (!ok) raise_timeout(&abort_sh, a.status);
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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
                      const CUtensorMap* tv, const CUtensorMap* to, cudaStream_t st, int grid,
                      int dev) {
  using Lay = Layout<D>;
  static std::atomic<bool> attrs_set[64];  // once per instantiation and device
  if (!attrs_set[dev].load()) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, kLse>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_tc_kernel<D, kLse>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attrs_set[dev].store(true);
  }
  const int slot = (int)(g_launches.fetch_add(1u) % kSchedRing);
  attn_tc_kernel<D, kLse><<<grid, kThreads, Lay::kSmem, st>>>(*tq, *tk, *tv, *to, a, slot);
  return cudaGetLastError();
}

}  // namespace

size_t tile_lists_bytes(int64_t n_items, int Lk) { return lists_bytes(n_items, Lk); }

cudaError_t launch_tile_lists(const AttnArgs& a, int32_t* lists, cudaStream_t st) {
  const int64_t n_items = (int64_t)a.B * a.H * ((a.L + kBM - 1) / kBM);
  tile_lists_kernel<<<(unsigned)((n_items + kListWarps - 1) / kListWarps), kListWarps * 32, 0,
                      st>>>(a, lists);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, const CUtensorMap* to, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_num_sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  // persistent CTAs, two per SM, each running one tile at a time
  const int64_t n_items = (int64_t)a.B * a.H * ((a.L + kBM - 1) / kBM);
  const int64_t cap = (int64_t)kCtasPerSm * g_num_sms[dev];
  const int grid = (int)(n_items < cap ? n_items : cap);
  if (a.d == 128)
    return a.lse ? launch_tc<128, true>(a, tq, tk, tv, to, st, grid, dev)
                 : launch_tc<128, false>(a, tq, tk, tv, to, st, grid, dev);
  return a.lse ? launch_tc<64, true>(a, tq, tk, tv, to, st, grid, dev)
               : launch_tc<64, false>(a, tq, tk, tv, to, st, grid, dev);
}

}  // namespace sdl
