// bf16 block-sparse / dense attention on sm_100a tensor cores.
//
// The fused IO-aware block-sparse kernel of the Step-dLLM abstract,
// re-designed for Blackwell.  A work item is a 128-row query tile of one
// head; it walks the kept key blocks of its rows, two 64-token sub-blocks
// (128 keys) per step.  CTAs are persistent (one per SM).  Each runs two
// independent item streams: the MMA issuer alternates between them, so one
// stream's softmax overlaps the other stream's products.  Items come from a
// global counter, first come first served (tiles differ in cost by the length
// of their kept lists).
//
//   warp 0        K producer: the K sub-blocks of every step by TMA
//                 (128-byte-swizzled 64x64 boxes) into a 2-deep ring, in the
//                 merged step order of the two streams (below); the Q tile of
//                 a stream's next item once that stream's last S product of
//                 the previous item has completed.
//   warp 2        V producer: the V sub-blocks, same order, own 2-deep ring.
//   warp 3        item producer: takes items, builds the union list of an
//                 item's two query blocks into a free list slot of whichever
//                 stream has one (two per stream) and prefetches its Q tile
//                 into L2.  Items whose lists are empty (only a caller's mask
//                 can have empty rows) are written here as zero rows.
//   warp 1        TMEM allocator and MMA issuer (one thread):
//                   S_t = Q_t K^T  tcgen05.mma kind::f16, A and B from shared
//                                  memory, M=128, N=128, fp32 in TMEM;
//                   O_t += P_t V   A = P_t (bf16, over S_t's first 64 TMEM
//                                  columns), B = V from shared memory
//                                  (N-major), M=128, N=d.
//                 A stream's next S is issued after its PV product (the two
//                 share S_t's columns), which also leaves O_t quiescent for
//                 that stream's softmax once the S product has completed.
//   warps 4-7     softmax of stream 0, warps 8-11 of stream 1: one thread per
//                 query row (its TMEM lane), all 128 columns of the step.
//                 Online softmax in the log2 domain; the running max is raised
//                 only when it grows by more than 8 (a factor 256), and O_t is
//                 rescaled in TMEM only then; P written back as bf16, the row
//                 sum taken over those rounded weights (the LSE's over the
//                 fp32 weights).  Epilogue per item: O / l rounded to bf16
//                 and written by TMA tensor stores from a per-warp
//                 shared-memory box, LSE.
//
// Merged step order: the producers and the MMA issuer take the steps of the
// two streams alternately (0, 1, 0, 1, ...); once a stream has no more items
// the other continues alone.  Each derives this order from the published
// lists, so the K and V rings are filled and drained in one order.
//
// With 64-token blocks a 128-row tile covers two query blocks; the item walks
// the union of their kept lists and masks, per 64x64 quadrant, the key
// sub-blocks a query block did not keep.  With 128-token blocks both halves
// share one list.  Dense attention is the same walk over every sub-block.
//
// TMEM (512 columns): S_0 at column 0, S_1 at 128, O_0 at 256, O_1 at 384.
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
constexpr int kStages = 2;       // K and V ring depth
constexpr int kStreams = 2;
constexpr int kSlots = 2;        // list slots per stream (at most 4)
constexpr int kMaxSub = 1024;    // 64-token sub-blocks per sequence (L <= 65536)
constexpr int kThreads = 384;    // 12 warps
constexpr int kKWarp = 0, kMmaWarp = 1, kVWarp = 2, kItemWarp = 3, kSoftWarp0 = 4;
constexpr int kBox = 64 * 128;   // bytes of one 64-row x 64-column bf16 box
constexpr int kOBoxBytes = 32 * 64;  // one 32-row x 32-column bf16 output box
constexpr uint32_t kTmemCols = 512;
// Of every 8 weights, how many take exp2_poly on the FMA pipe instead of
// MUFU.EX2 (even values; the step is issue-bound more than MUFU-bound here,
// and 0 measured fastest).
constexpr int kPolyPer8 = 0;

__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * (uint32_t)t; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * (uint32_t)t; }

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;           // 128-byte column chunks
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;     // one stage of K (or V)
  static constexpr int kChunkRowsQ = kBM * 128;    // bytes per Q column chunk
  static constexpr int kChunkRowsKV = kBN * 128;   // bytes per K/V column chunk
  static constexpr int kOffQ = 0;                  // one Q tile per stream
  static constexpr int kOffK = kStreams * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  // output staging: per softmax warp one 32-row x 32-column bf16 box
  // (64-byte rows, 64-byte swizzle) for the tensor stores of O
  static constexpr int kOffO = kOffV + kStages * kKVBytes;
  static constexpr int kBytes = kOffO + 8 * kOBoxBytes;
  static constexpr int kSmem = kBytes + 1024;      // + alignment slack
};

// Consumers of a list slot: K producer, V producer, MMA, the stream's 4 softmax warps.
constexpr int kListConsumers = 3 + 4;

struct Bars {
  uint64_t list_full[kStreams][kSlots];   // slot published by the item producer
  uint64_t list_empty[kStreams][kSlots];  // slot released by every consumer
  uint64_t q_full[kStreams];
  uint64_t q_empty[kStreams];  // the S products of the stream's item completed
  uint64_t s_full[kStreams];   // S_t written
  uint64_t p_full[kStreams];   // P_t written (one arrival per softmax warp)
  uint64_t o_full[kStreams];   // every product of the stream's item completed
  uint64_t kfull[kStages], kempty[kStages];
  uint64_t vfull[kStages], vempty[kStages];
  uint64_t done;
};

// One published item: its kept list, sub-block index | keep bits << 16
// (bit 0: query rows 0..63 keep it, bit 1: rows 64..127).
struct Slot {
  int item;  // -1: end of the stream
  int n_ent;
  int b, h;
  int t0, t1;  // first tokens of the tile's two 64-row halves (L: half unused)
  uint32_t ent[kMaxSub];
};

// Step records, written by the K producer for the MMA issuer, one per step
// of the merged order (ring position g % kCmdRing):
//   bit 0 stream, bit 1 first step of its item, bit 2 last step of its item,
//   bits 3-4 the item's list slot, bits 5-6 distance back to the stream's
//   previous step in the merged order (0: none), bit 7 end of the order.
constexpr int kCmdRing = 8;
constexpr uint32_t kCmdEnd = 0x80u;

// Item counters of in-flight launches.  Launch n uses entry n % kSchedRing;
// its CTAs take items with atomicAdd on `next`, and the last CTA to finish
// puts the entry back to zero for a later launch.
constexpr int kSchedRing = 64;
struct Sched {
  unsigned next;
  unsigned finished;
};
__device__ Sched g_sched[kSchedRing];

// A single-thread consumer's position in the merged step order.
struct Cursor {
  int k0, k1;  // ordinal of each stream's current item (-1: none yet)
  int j0, j1;  // next step of that item
  int n0, n1;  // steps of that item
  bool live0, live1;
  int turn;
  __device__ void init() {
    k0 = k1 = -1;
    j0 = j1 = n0 = n1 = 0;
    live0 = live1 = true;
    turn = 0;
  }
  __device__ int k(int t) const { return t ? k1 : k0; }
  __device__ bool live(int t) const { return t ? live1 : live0; }
  __device__ bool at_end(int t) const { return t ? j1 == n1 : j0 == n0; }
  __device__ void open(int t, int k_, int n_) {
    if (t) {
      k1 = k_;
      j1 = 0;
      n1 = n_;
    } else {
      k0 = k_;
      j0 = 0;
      n0 = n_;
    }
  }
  __device__ void kill(int t) {
    if (t)
      live1 = false;
    else
      live0 = false;
  }
  // consumes stream t's next step: returns its index within the item
  __device__ int take(int t) {
    turn = t ^ 1;
    return t ? j1++ : j0++;
  }
};

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

template <int D, bool kLse>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                   AttnArgs a, int sched_slot) {
  using Lay = Layout<D>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                            ~(uintptr_t)1023);
  __shared__ Bars bars;
  __shared__ Slot slots[kStreams][kSlots];
  __shared__ uint32_t bmask[2][kMaxSub / 32];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_sh;
  __shared__ uint32_t cmd[kCmdRing];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = (a.L + kBM - 1) / kBM;
  const int n_items = a.B * a.H * n_qt;

  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int t = 0; t < kStreams; ++t) {
        for (int s = 0; s < kSlots; ++s) {
          mbar_init(&bars.list_full[t][s], 1);
          mbar_init(&bars.list_empty[t][s], kListConsumers);
        }
        mbar_init(&bars.q_full[t], 1);
        mbar_init(&bars.q_empty[t], 1);
        mbar_init(&bars.s_full[t], 1);
        mbar_init(&bars.p_full[t], 4);
        mbar_init(&bars.o_full[t], 1);
      }
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&bars.kfull[s], 1);
        mbar_init(&bars.kempty[s], 1);
        mbar_init(&bars.vfull[s], 1);
        mbar_init(&bars.vempty[s], 1);
      }
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

  // (The producer and MMA roles run warp-converged; one elected lane issues
  // their copies, MMAs and arrivals, and every wait is made warp-uniform.)
  // Stream of the next step in the merged order, opening that stream's next
  // item when its current one is used up (on_open(t) runs then); -1 once both
  // streams have ended, -2 on timeout.  If blocked(t), the caller cannot take
  // a step of stream t yet: t is returned and nothing is opened.
  auto peek = [&](Cursor& C, auto&& blocked, auto&& on_open) -> int {
    for (int attempt = 0; attempt < 2; ++attempt) {
      const int t = C.turn ^ attempt;
      if (!C.live(t)) continue;
      if (blocked(t)) return t;
      if (C.at_end(t)) {
        const int kn = C.k(t) + 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.list_full[t][kn % kSlots], (kn / kSlots) & 1,
                                                &abort_sh, a.status, kWaitLimitNs)))
          return -2;
        const Slot& S = slots[t][kn % kSlots];
        if (S.item < 0) {
          C.kill(t);
          continue;
        }
        C.open(t, kn, (S.n_ent + 1) / 2);
        if (!on_open(t)) return -2;
      }
      return t;
    }
    return -1;
  };

  if (warp == kItemWarp) {
    // ====================================================== item producer
    const int nsub = a.Lk / kSubBlock;
    int pub0 = 0, pub1 = 0;  // slots published per stream (end marker included)
    bool ended0 = false, ended1 = false;
    bool exhausted = false;  // the launch's counter ran out
    bool ok = true;
    uint64_t t_idle = 0;
    while (ok && !(ended0 && ended1)) {
      bool progressed = false;
#pragma unroll 1
      for (int t = 0; t < kStreams; ++t) {
        if (t ? ended1 : ended0) continue;
        const int pub = t ? pub1 : pub0;
        const int slot = pub % kSlots;
        bool free_slot = pub < kSlots;
        if (!free_slot) {
          if (lane == 0)
            free_slot = mbar_test_wait(&bars.list_empty[t][slot], ((pub / kSlots) - 1) & 1);
          free_slot = __shfl_sync(0xffffffffu, free_slot ? 1 : 0, 0) != 0;
        }
        if (!free_slot) continue;
        progressed = true;
        Slot& S = slots[t][slot];
        // take items until a non-empty one (or none is left)
        int item = -1, n_ent = 0, b = 0, h = 0, t0 = 0, t1 = 0;
        while (!exhausted) {
          unsigned taken = 0;
          if (lane == 0) taken = atomicAdd(&g_sched[sched_slot].next, 1u);
          taken = __shfl_sync(0xffffffffu, taken, 0);
          if (taken >= (unsigned)n_items) {
            exhausted = true;
            break;
          }
          item = (int)taken;
          if (a.order != nullptr) {
            // costliest tiles first (the order is a permutation of the items)
            const int o = a.order[item];
            if (o < 0 || o >= n_items) {
              atomicOr(a.status, kDevBadMask);
              continue;
            }
            item = o;
          }
          b = item / (a.H * n_qt);
          h = (item / n_qt) % a.H;
          if (a.plan != nullptr) {
            // the tile's two query blocks from the plan (64-token blocks)
            const int qb0 = a.plan[2 * (int64_t)item], qb1 = a.plan[2 * (int64_t)item + 1];
            if (qb0 >= a.nb || qb0 < -1 || qb1 >= a.nb || qb1 < -1)
              atomicOr(a.status, kDevBadMask);
            t0 = (qb0 >= 0 && qb0 < a.nb) ? qb0 * 64 : a.L;
            t1 = (qb1 >= 0 && qb1 < a.nb) ? qb1 * 64 : a.L;
          } else {
            t0 = (item % n_qt) * kBM;
            t1 = t0 + 64 < a.L ? t0 + 64 : a.L;
          }
          // kept 64-token key sub-blocks of the two query halves, as bitmaps
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
                if (bad_range || (x > beg && a.col_idx[x - 1] >= jb))
                  atomicOr(a.status, kDevBadMask);
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
          n_ent = __shfl_sync(0xffffffffu, incl, 31);
          __syncwarp();
          if (n_ent == 0) {
            write_empty_tile<D>(a, b, h, t0, t1, lane);
            __syncwarp();
            continue;
          }
          int pos = incl - c;
          for (uint32_t mb = wu; mb; mb &= mb - 1) {
            const int bit = __ffs(mb) - 1;
            const uint32_t keep = ((w0 >> bit) & 1u) | (((w1 >> bit) & 1u) << 1);
            S.ent[pos++] = (uint32_t)(lane * 32 + bit) | (keep << 16);
          }
          break;
        }
        const bool end_marker = n_ent == 0;  // (only when the counter ran out)
        if (lane == 0) {
          if (end_marker) {
            S.item = -1;
            S.n_ent = 0;
          } else {
            S.item = item;
            S.n_ent = n_ent;
            S.b = b;
            S.h = h;
            S.t0 = t0;
            S.t1 = t1;
            // its Q tile is loaded when this stream's previous item is done; warm L2 now
            for (int cc = 0; cc < Lay::kChunks; ++cc)
              for (int s = 0; s < 2; ++s)
                if ((s ? t1 : t0) < a.L) tma_prefetch_l2_4d(&tmq, cc * 64, s ? t1 : t0, h, b);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.list_full[t][slot]);
        if (t) {
          ++pub1;
          ended1 = end_marker;
        } else {
          ++pub0;
          ended0 = end_marker;
        }
      }
      if (progressed) {
        t_idle = 0;
      } else {
        // every slot of both streams is busy: back off, bounded by the wait limit
        if (t_idle == 0) t_idle = globaltimer_ns();
        __nanosleep(500);
        if (abort_sh || globaltimer_ns() - t_idle > kWaitLimitNs) ok = false;
      }
    }
    if (lane == 0 && !ok) raise_timeout(&abort_sh, a.status);
  } else if (warp == kKWarp || warp == kVWarp) {
    // ================================================= K and V producers
    const bool isk = warp == kKWarp;
    uint64_t* full = isk ? bars.kfull : bars.vfull;
    uint64_t* empty = isk ? bars.kempty : bars.vempty;
    const CUtensorMap* tm = isk ? &tmk : &tmv;
    uint8_t* ring = dsm + (isk ? Lay::kOffK : Lay::kOffV);
    const int group = a.H / a.Hkv;
    {
      const bool leader = elect_one_sync();
      if (leader) {
        prefetch_tensormap(tm);
        if (isk) prefetch_tensormap(&tmq);
      }
      Cursor C;
      C.init();
      int qiss0 = 0, qiss1 = 0;  // Q tiles loaded per stream
      int last_g0 = -1, last_g1 = -1;  // merged position of each stream's previous step
      bool ok = true;
      int g = 0;  // position in the merged order: ring stage g % kStages
      auto never = [](int) { return false; };
      auto on_open = [&](int t) -> bool {
        if (!isk) return true;
        // Q of the stream's new item, once its previous item's S products completed
        const int n = t ? qiss1 : qiss0;
        if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars.q_empty[t], (n - 1) & 1, &abort_sh,
                                                        a.status, kWaitLimitNs)))
          return false;
        const Slot& S = slots[t][C.k(t) % kSlots];
        uint8_t* sq = dsm + Lay::kOffQ + t * Lay::kQBytes;
        if (leader) {
          mbar_arrive_expect_tx(&bars.q_full[t], Lay::kQBytes);
          for (int cc = 0; cc < Lay::kChunks; ++cc)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(sq + cc * Lay::kChunkRowsQ + s * kBox, &tmq, &bars.q_full[t], cc * 64,
                          s ? S.t1 : S.t0, S.h, S.b);
        }
        if (t)
          ++qiss1;
        else
          ++qiss0;
        return true;
      };
      for (;;) {
        const int t = peek(C, never, on_open);
        if (t == -2) ok = false;
        if (t < 0) break;
        const int jj = C.take(t);
        const int slot = C.k(t) % kSlots;
        const Slot& S = slots[t][slot];
        const int n_ent = S.n_ent;
        const uint32_t e0 = S.ent[2 * jj];
        const uint32_t e1 = (2 * jj + 1 < n_ent) ? S.ent[2 * jj + 1] : e0;
        const int sub0 = (int)(e0 & 0xFFFFu), sub1 = (int)(e1 & 0xFFFFu);
        const int kh = S.h / group, b = S.b;
        const int st = g % kStages;
        if (g >= kStages &&
            !(ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ((g / kStages) - 1) & 1,
                                                     &abort_sh, a.status, kWaitLimitNs))))
          break;
        uint8_t* dst = ring + st * Lay::kKVBytes;
        if (isk) {
          const int prev = t ? last_g1 : last_g0;
          const uint32_t rec = (uint32_t)t | (jj == 0 ? 2u : 0u) | (C.at_end(t) ? 4u : 0u) |
                               ((uint32_t)slot << 3) | ((uint32_t)(prev < 0 ? 0 : g - prev) << 5);
          if (t)
            last_g1 = g;
          else
            last_g0 = g;
          if (leader) cmd[g % kCmdRing] = rec;  // published by the arrive below
        }
        if (leader) {
          mbar_arrive_expect_tx(&full[st], Lay::kKVBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, tm, &full[st], c * 64,
                          (s ? sub1 : sub0) * kSubBlock, kh, b);
          if (C.at_end(t)) mbar_arrive(&bars.list_empty[t][slot]);
        }
        ++g;
      }
      if (leader) {
        if (!ok) raise_timeout(&abort_sh, a.status);
        // Drain: every copy issued above lands before the CTA exits.
        volatile int no_abort = 0;
        for (int st = (g > kStages ? g - kStages : 0); st < g; ++st)
          if (!mbar_wait(&full[st % kStages], (st / kStages) & 1, &no_abort, nullptr,
                         kWaitLimitNs))
            atomicOr(a.status, kDevTimeout);
        if (qiss0 > 0 &&
            !mbar_wait(&bars.q_full[0], (qiss0 - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
        if (qiss1 > 0 &&
            !mbar_wait(&bars.q_full[1], (qiss1 - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
      }
      __syncwarp();
      if (isk && ok) {
        // End of the merged order: an end record, published through the next
        // stage's full barrier once that stage is free (a plain arrival, no
        // bytes).  It comes after the drain above, whose waits name the
        // phases of the last copies.
        const int st = g % kStages;
        if (g >= kStages)
          ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ((g / kStages) - 1) & 1, &abort_sh,
                                                 a.status, kWaitLimitNs));
        if (ok && leader) {
          cmd[g % kCmdRing] = kCmdEnd;
          mbar_arrive(&full[st]);
        }
        if (!ok && leader) raise_timeout(&abort_sh, a.status);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA
    // Steps come as records in the merged order.  S of step s may be issued
    // once the PV product of its stream's previous step has been (the two
    // share S_t's columns); at most two S products run ahead of the PVs.
    {
      const bool leader = elect_one_sync();
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kBM, D, true);
      // Descriptors are built once: the start-address field (bits 0..13,
      // address >> 4) of the descriptor for address x + off is the base
      // descriptor's plus off >> 4, without carry (shared addresses < 2^18).
      const uint64_t dq = smem_desc_sw128(smem_u32(dsm + Lay::kOffQ), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_u32(dsm + Lay::kOffK), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(dsm + Lay::kOffV), Lay::kChunkRowsKV, 1024);
      int nq0 = 0, nq1 = 0;  // Q tiles consumed per stream
      int np0 = 0, np1 = 0;  // PV products issued per stream
      int p = 0;             // next PV (merged position)
      int s = 0;             // next S (merged position)
      bool s_end = false;    // the end record has been read
      uint32_t s_rec = 0;    // record of step s, once read
      bool s_read = false;
      bool ok = true;
      // Issues S of step s if its record allows it now: 1 issued, 0 not now.
      auto try_s = [&]() -> int {
        if (s_end || s >= p + 2) return 0;
        const int st = s % kStages;
        if (!s_read) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.kfull[st], (s / kStages) & 1,
                                                       &abort_sh, a.status, kWaitLimitNs))))
            return 0;
          s_rec = cmd[s % kCmdRing];
          s_read = true;
          if (s_rec & kCmdEnd) {
            s_end = true;
            return 0;
          }
        }
        const int gap = (int)((s_rec >> 5) & 3u);
        if (gap > 0 && s - gap >= p) return 0;  // that stream's PV is not issued yet
        const int t = (int)(s_rec & 1u);
        if (s_rec & 2u) {  // first step of an item: its Q tile
          const int n = t ? nq1 : nq0;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.q_full[t], n & 1, &abort_sh,
                                                       a.status, kWaitLimitNs))))
            return 0;
          if (t)
            ++nq1;
          else
            ++nq0;
        }
        tc_fence_after();
        const uint64_t ad0 = dq + (uint64_t)((t * Lay::kQBytes) >> 4);
        const uint64_t bd0 = dk + (uint64_t)((st * Lay::kKVBytes) >> 4);
        const uint32_t dcol = tmem + col_s(t);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 d-columns: chunk kk / 4, 32 bytes (kk % 4) inside the swizzle atom
          const uint64_t offq = (uint64_t)(((kk / 4) * Lay::kChunkRowsQ + (kk % 4) * 32) >> 4);
          const uint64_t offk = (uint64_t)(((kk / 4) * Lay::kChunkRowsKV + (kk % 4) * 32) >> 4);
          if (leader) mma_bf16_ss(dcol, ad0 + offq, bd0 + offk, idS, kk > 0 ? 1u : 0u);
        }
        if (leader) {
          tc_commit(&bars.kempty[st]);
          tc_commit(&bars.s_full[t]);
          if (s_rec & 4u) tc_commit(&bars.q_empty[t]);
        }
        ++s;
        s_read = false;
        return 1;
      };
      while (ok && try_s() == 1) {
      }
      while (ok && p < s) {
        // O_t += P_t V for step p
        const uint32_t rec = cmd[p % kCmdRing];
        const int t = (int)(rec & 1u);
        const int np = t ? np1 : np0;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.p_full[t], np & 1, &abort_sh,
                                                     a.status, kWaitLimitNs))))
          break;
        const int st = p % kStages;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.vfull[st], (p / kStages) & 1,
                                                     &abort_sh, a.status, kWaitLimitNs))))
          break;
        tc_fence_after();
        const uint64_t bd0 = dv + (uint64_t)((st * Lay::kKVBytes) >> 4);
        const uint32_t pcol = tmem + col_s(t);
        const uint32_t ocol = tmem + col_o(t);
        const bool first = (rec & 2u) != 0;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // keys [16 kk, 16 kk + 16): V rows 16 kk.. (128 bytes each); P elements
          // packed in columns [8 kk, 8 kk + 8)
          if (leader)
            mma_bf16_ts(ocol, pcol + 8 * kk, bd0 + (uint64_t)((kk * 16 * 128) >> 4), idPV,
                        (!first || kk > 0) ? 1u : 0u);
        }
        if (leader) {
          tc_commit(&bars.vempty[st]);
          if (rec & 4u) {
            tc_commit(&bars.o_full[t]);
            mbar_arrive(&bars.list_empty[t][(rec >> 3) & 3u]);
          }
        }
        ++p;
        if (t)
          ++np1;
        else
          ++np0;
        while (ok && try_s() == 1) {
        }
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
    }
  } else {
    // ============================================================ softmax
    const int t = (warp - kSoftWarp0) / 4;  // stream
    const int quad = warp & 3;              // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t scol = trow + col_s(t);
    const uint32_t ocol = trow + col_o(t);
    uint8_t* ostage = dsm + Lay::kOffO + (warp - kSoftWarp0) * kOBoxBytes;
    const float sl2 = a.scale_log2;
    int n = 0;  // steps of this stream so far
    bool ok = true;
    for (int k = 0;; ++k) {
      const int slot = k % kSlots;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.list_full[t][slot], (k / kSlots) & 1,
                                             &abort_sh, a.status, kWaitLimitNs));
      if (!ok) break;
      const Slot& S = slots[t][slot];
      if (S.item < 0) break;
      const int n_ent = S.n_ent, b = S.b, h = S.h, tok = (half ? S.t1 : S.t0) + (row & 63);
      const int n_steps = (n_ent + 1) / 2;
      float m = -INFINITY;  // running max (log2 units) used as the exponent reference
      float l = 0.f;        // row sum of the bf16-rounded weights
      float lx = 0.f;       // row sum of the unrounded weights (LSE only)
      for (int j = 0; j < n_steps; ++j, ++n) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[t], n & 1, &abort_sh, a.status,
                                               kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t e0 = S.ent[2 * j];
        const uint32_t e1 = (2 * j + 1 < n_ent) ? S.ent[2 * j + 1] : (e0 & 0xFFFFu);
        // (keep is uniform over a warp: its 32 rows lie in one query block)
        const bool keep0 = (e0 >> (16 + half)) & 1u;
        const bool keep1 = (e1 >> (16 + half)) & 1u;
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
            // O_t is quiescent: this step's S product was issued after the
            // stream's previous PV product and has completed.
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
        // bf16 pairs over S_t's first 64 columns; l sums the rounded weights
        // (pair arithmetic packed: x = s * scale_log2 - m, row sums)
        const uint64_t sl2x2 = pack2(sl2, sl2), nmx2 = pack2(-m, -m);
        uint64_t rs2 = pack2(0.f, 0.f), rx2 = pack2(0.f, 0.f);
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
              float p0, p1;
              if ((x & 7) < 8 - kPolyPer8) {
                p0 = ex2_approx(xv.x);
                p1 = ex2_approx(xv.y);
              } else {
                const float2 e = exp2_poly2(xv.x, xv.y);
                p0 = e.x;
                p1 = e.y;
              }
              __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
              const uint32_t u = *reinterpret_cast<uint32_t*>(&pk);
              rs2 = add2(rs2, pack2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u)));
              if constexpr (kLse) rx2 = add2(rx2, pack2(p0, p1));
              pw[x / 2] = u;
            }
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) pw[x] = 0u;
          }
          tmem_st16(scol + 16 * c, pw);
        }
        {
          const float2 a2 = unpack2(rs2), b2 = unpack2(rx2);
          l += a2.x + a2.y;
          lx += b2.x + b2.y;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[t]);
      }
      if (!ok) break;
      // --------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.o_full[t], k & 1, &abort_sh, a.status,
                                             kWaitLimitNs));
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
      if (lane == 0) mbar_arrive(&bars.list_empty[t][slot]);
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
                      const CUtensorMap* tv, const CUtensorMap* to, cudaStream_t st, int grid) {
  using Lay = Layout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, kLse>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
  if (e != cudaSuccess) return e;
  const int slot = (int)(g_launches.fetch_add(1u) % kSchedRing);
  attn_tc_kernel<D, kLse><<<grid, kThreads, Lay::kSmem, st>>>(*tq, *tk, *tv, *to, a, slot);
  return cudaGetLastError();
}

}  // namespace

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
  // one persistent CTA per SM (the shared-memory footprint admits one), each
  // running two tiles at a time
  const int64_t n_items = (int64_t)a.B * a.H * ((a.L + kBM - 1) / kBM);
  const int64_t want = (n_items + kStreams - 1) / kStreams;
  const int grid = (int)(want < g_num_sms[dev] ? want : g_num_sms[dev]);
  if (a.d == 128)
    return a.lse ? launch_tc<128, true>(a, tq, tk, tv, to, st, grid)
                 : launch_tc<128, false>(a, tq, tk, tv, to, st, grid);
  return a.lse ? launch_tc<64, true>(a, tq, tk, tv, to, st, grid)
               : launch_tc<64, false>(a, tq, tk, tv, to, st, grid);
}

}  // namespace sdl
