// bf16 block-sparse / dense attention on sm_100a tensor cores.
//
// The fused IO-aware block-sparse kernel of the Step-dLLM abstract,
// re-designed for Blackwell.  A work item is a 128-row query tile of one
// head; it walks the kept key blocks of its rows, two 64-token sub-blocks
// (128 keys) per step.  CTAs are persistent, one per SM, and take items from
// a global counter, first come first served (tiles differ in cost by the
// length of their kept lists).
//
// Each step's 128 keys are split between two softmax warpgroups: group 0
// owns keys 0..63 (the step's first sub-block), group 1 keys 64..127.  Each
// group runs its own online softmax over its half of every step, with its own
// running maximum, row sums and O accumulator in TMEM, so the two groups never
// wait on each other inside a tile; the epilogue merges the two partial
// results (the same merge as for two key ranges of a split softmax).  S is
// double-buffered in TMEM, so the product S(n+1) = Q K(n+1)^T runs on the
// tensor cores while both groups work on S(n).
//
//   warp 0        loads: takes items and copies an item's prebuilt list
//                 (tile_lists_kernel, run once per mask) or builds the union
//                 list of its two query blocks into a list slot (three slots,
//                 the next item's list while the current item runs); per item
//                 its Q tile into one of two Q stages, per step its K and V
//                 sub-blocks by TMA (128-byte-swizzled 64x64 boxes) into
//                 two-stage K and V rings, K one step ahead of V.  Items whose
//                 lists are empty (only a caller's mask can have empty rows)
//                 are written here as zero rows.
//   warp 1        TMEM allocator and MMA issuer (one elected thread):
//                   S(n) = Q K(n)^T  tcgen05.mma kind::f16, A and B from shared
//                                    memory, M=128, N=128, fp32 into TMEM
//                                    buffer n % 2;
//                   O_g += P_g V_g   for each group g once it has written its
//                                    weights: A = P_g (bf16 in TMEM, over the
//                                    group's own S columns), B = the group's 64
//                                    V rows (N-major), M=128, N=d.
//                 Issue order S(n), O(n-1): the next S is on the tensor pipe
//                 before the groups finish the current step.
//   warps 2-5     softmax group 0, warps 6-9 group 1: one thread per query row
//                 (its TMEM lane quadrant), 64 columns of each step.  Online
//                 softmax in the log2 domain; the running maximum is raised only
//                 when it grows by more than 8 (a factor 256), and the group's O
//                 is rescaled in TMEM only then; P written back as bf16, the row
//                 sum taken over those rounded weights (the LSE's over the fp32
//                 weights).  Epilogue per item: the groups exchange their row
//                 maxima and sums through shared memory, each merges and scales
//                 half of O's columns, rounds to bf16 and writes them by TMA
//                 tensor stores from per-warp shared-memory boxes; group 0
//                 writes the LSE.
//
// With 64-token blocks a 128-row tile covers two query blocks; the item walks
// the union of their kept lists and masks, per 64x64 quadrant, the key
// sub-blocks a query block did not keep.  With 128-token blocks both halves
// share one list.  Dense attention is the same walk over every sub-block.
//
// TMEM (512 columns, the whole SM's): S buffers at columns 0 and 128 (group g
// reads columns 64 g .. 64 g + 63 of a buffer and writes its P over the first 32
// of them), O of group g at 256 + 128 g.
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
constexpr int kGroups = 2;       // softmax warpgroups (one per 64-key half of a step)
constexpr int kSoftWarps = 4 * kGroups;
constexpr int kThreads = 32 * (2 + kSoftWarps);  // load, MMA, softmax
constexpr int kLoadWarp = 0, kMmaWarp = 1, kSoftWarp0 = 2;
constexpr int kQStages = 2, kKStages = 2, kVStages = 2;
constexpr int kBox = 64 * 128;   // bytes of one 64-row x 64-column bf16 box
constexpr int kOBoxBytes = 32 * 64;  // one 32-row x 32-column bf16 output box
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S buffer b at kColS + 128 b
constexpr uint32_t kColO = 256;  // O of group g at kColO + 128 g
// The reference maximum of a row is raised (and O rescaled) only when the
// tile maximum exceeds it by more than this many log2 units.
constexpr float kRaiseLog2 = 16.0f;

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;           // 128-byte column chunks
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;     // one stage of K (or V)
  static constexpr int kChunkRowsQ = kBM * 128;    // bytes per Q column chunk
  static constexpr int kChunkRowsKV = kBN * 128;   // bytes per K/V column chunk
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQStages * kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  // output staging: per softmax warp one 32-row x 32-column bf16 box
  // (64-byte rows, 64-byte swizzle) for the tensor stores of O
  static constexpr int kOffO = kOffV + kVStages * kKVBytes;
  static constexpr int kBytes = kOffO + kSoftWarps * kOBoxBytes;
  static constexpr int kSmem = kBytes + 1024;      // + alignment slack
};
// one CTA per SM: 228 KB of shared memory per SM, 1 KB of it reserved per
// CTA, and up to 12 KB of static shared memory
static_assert(Layout<128>::kSmem + 12 * 1024 + 1024 <= 228 * 1024, "shared memory");

// Consumers of a list slot: the MMA warp and the softmax warps.
constexpr int kListConsumers = 1 + kSoftWarps;

struct Bars {
  uint64_t list_full[kSlots];   // slot published by the load warp
  uint64_t list_empty[kSlots];  // slot released by every consumer
  uint64_t q_full[kQStages], q_empty[kQStages];  // Q landed / the item's S products completed
  uint64_t kfull[kKStages], kempty[kKStages];
  uint64_t vfull[kVStages], vempty[kVStages];
  uint64_t s_full[2];           // S buffer b written
  uint64_t p_ready[kGroups][2]; // group g's P in buffer b written (one arrival per warp)
  uint64_t pv_done[kGroups][2]; // group g's product of a step of parity b completed
  uint64_t o_full;              // every product of the item completed
  uint64_t o_empty;             // the epilogue has read O (one arrival per softmax warp)
  uint64_t xch;                 // the groups' row maxima and sums exchanged
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
// its CTAs take items with atomicAdd on `next` (each CTA's last add is the
// one past the end), and the last CTA to finish checks that the counter saw
// exactly the launch's items and one add per CTA past them -- more means
// another launch in flight shared the entry -- then puts it back to zero.
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
    if (qb0 >= a.nb || qb0 < -1 || qb1 >= a.nb || qb1 < -1)
      report_bad_mask(a.status, kBadPlanEntry, item);
    t0 = (qb0 >= 0 && qb0 < a.nb) ? qb0 * 64 : a.L;
    t1 = (qb1 >= 0 && qb1 < a.nb) ? qb1 * 64 : a.L;
  } else {
    t0 = (item % n_qt) * kBM;
    t1 = t0 + 64 < a.L ? t0 + 64 : a.L;
  }
}

// The kept 64-token key sub-blocks of a tile's two query halves, as bitmaps
// in `bmask` (all key sub-blocks without a mask), listed with their keep
// bits into `ent` (shared or global memory) in the order below; all lanes of
// one warp.  Returns the list's length.
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
        if (bad_range || (x > beg && a.col_idx[x - 1] >= jb))
          report_bad_mask(a.status, kBadListEntry, jb);
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
  // The union with per-half keep bits, ordered for the two softmax groups: a
  // step's first entry goes to group 0, its second to group 1, and a query
  // block's rows sit in two of the four lane quadrants (two SMSPs).  A step
  // pairing an entry only the first query block keeps (A) with one only the
  // second keeps (B) gives every SMSP one busy warp; any other pair loads two
  // SMSPs with two.  So the first min(|A|, |B|) steps pair A with B; the
  // unpaired rest of A or B follows, then the entries both keep (C), each class
  // in ascending sub-block order.  Lane w handles bitmap word w.
  const uint32_t w0 = bmask[0][lane], w1 = bmask[1][lane];
  const uint32_t wa = w0 & ~w1, wb = w1 & ~w0, wc = w0 & w1;
  int ia = __popc(wa), ib = __popc(wb), ic = __popc(wc);  // inclusive prefix sums
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, ia, o);
    const int vb = __shfl_up_sync(0xffffffffu, ib, o);
    const int vc = __shfl_up_sync(0xffffffffu, ic, o);
    if (lane >= o) {
      ia += va;
      ib += vb;
      ic += vc;
    }
  }
  const int na = __shfl_sync(0xffffffffu, ia, 31), nb_ = __shfl_sync(0xffffffffu, ib, 31);
  const int nc = __shfl_sync(0xffffffffu, ic, 31);
  const int np = na < nb_ ? na : nb_;           // A-B pairs
  const int rest = 2 * np + (na - np) + (nb_ - np);  // where C starts
  int ra = ia - __popc(wa), rb = ib - __popc(wb), rc = ic - __popc(wc);  // exclusive ranks
  for (uint32_t mb = w0 | w1; mb; mb &= mb - 1) {
    const int bit = __ffs(mb) - 1;
    const uint32_t keep = ((w0 >> bit) & 1u) | (((w1 >> bit) & 1u) << 1);
    int pos;
    if (keep == 1u) {
      pos = ra < np ? 2 * ra : 2 * np + (ra - np);
      ++ra;
    } else if (keep == 2u) {
      pos = rb < np ? 2 * rb + 1 : 2 * np + (na - np) + (rb - np);
      ++rb;
    } else {
      pos = rest + rc;
      ++rc;
    }
    ent[pos] = (uint16_t)((uint32_t)(lane * 32 + bit) | (keep << kKeepShift));
  }
  __syncwarp();
  return na + nb_ + nc;
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
        if (lane == 0) report_bad_mask(a.status, kBadRecord, item);
        continue;
      }
      b = item / (a.H * n_qt);
      h = (item / n_qt) % a.H;
      t0 = rec.z;
      t1 = rec.w;
      if (t0 < 0 || t0 > a.L || t1 < 0 || t1 > a.L) {
        if (lane == 0) report_bad_mask(a.status, kBadRecordRows, t0);
        continue;
      }
      const uint16_t* src = reinterpret_cast<const uint16_t*>(a.lists + (int64_t)n_items *
                                                                            kListRecInts) +
                            (int64_t)taken * lists_cap(a.Lk);
      for (int x = lane; x < n_ent; x += 32) {
        uint16_t e = src[x];
        if ((int)(e & kSubMask) >= nsub) {
          report_bad_mask(a.status, kBadRecordEntry, e);
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
          if (lane == 0) report_bad_mask(a.status, kBadOrderEntry, o);
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
        report_bad_mask(a.status, kBadListsOrder, item);
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


// Maximum of 32 fp32 logits (three-input max).
__device__ __forceinline__ float max32(const uint32_t* r) {
  float m0 = __uint_as_float(r[0]), m1 = __uint_as_float(r[1]);
#pragma unroll
  for (int x = 2; x < 30; x += 4) {
    m0 = max3f(m0, __uint_as_float(r[x]), __uint_as_float(r[x + 1]));
    m1 = max3f(m1, __uint_as_float(r[x + 2]), __uint_as_float(r[x + 3]));
  }
  return max3f(m0, m1, fmaxf(__uint_as_float(r[30]), __uint_as_float(r[31])));
}

// Softmax weights of 32 logits: p = exp2(s * scale_log2 - m) (x packed in
// pairs), rounded to bf16 pairs into pw[0..15]; rsa / rsb sum the rounded
// weights, each bf16 half added to an fp32 sum by one mixed-precision add;
// rx2 sums the unrounded ones (the LSE's).
template <bool kLse>
__device__ __forceinline__ void weights32(const uint32_t* r, uint64_t sl2x2, uint64_t nmx2,
                                          uint32_t* pw, float& rsa, float& rsb, uint64_t& rx2) {
#pragma unroll
  for (int x = 0; x < 32; x += 2) {
    const float2 xv =
        unpack2(fma2(pack2(__uint_as_float(r[x]), __uint_as_float(r[x + 1])), sl2x2, nmx2));
    const float p0 = ex2_approx(xv.x), p1 = ex2_approx(xv.y);
    __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
    const uint32_t u = *reinterpret_cast<uint32_t*>(&pk);
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(rsa), "+f"(rsb) : "r"(u));
    if constexpr (kLse) rx2 = add2(rx2, pack2(p0, p1));
    pw[x / 2] = u;
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
  __shared__ Slot slots[kSlots];
  __shared__ uint32_t bmask[2][kMaxSub / 32];
  // the groups' final row maxima (log2 units), sums of the rounded weights and
  // sums of the unrounded weights, exchanged at the epilogue
  __shared__ float xm[kGroups][kBM], xl[kGroups][kBM], xlx[kGroups][kBM];
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
      for (int s = 0; s < kQStages; ++s) {
        mbar_init(&bars.q_full[s], 1);
        mbar_init(&bars.q_empty[s], 1);
      }
      for (int s = 0; s < kKStages; ++s) {
        mbar_init(&bars.kfull[s], 1);
        mbar_init(&bars.kempty[s], 1);
      }
      for (int s = 0; s < kVStages; ++s) {
        mbar_init(&bars.vfull[s], 1);
        mbar_init(&bars.vempty[s], 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bars.s_full[b], 1);
        for (int g = 0; g < kGroups; ++g) {
          mbar_init(&bars.p_ready[g][b], 4);
          mbar_init(&bars.pv_done[g][b], 1);
        }
      }
      mbar_init(&bars.o_full, 1);
      mbar_init(&bars.o_empty, kSoftWarps);
      mbar_init(&bars.xch, kSoftWarps);
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
    int nk = 0;      // K copies issued (one per step)
    int nv = 0;      // V copies issued (one per step, one step behind K)
    // the step whose V is still to be loaded: its two sub-blocks, KV head, batch
    bool v_pend = false;
    int pv_sub0 = 0, pv_sub1 = 0, pv_kh = 0, pv_b = 0;
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
    // V of the pending step, once the product that last read its stage has completed
    auto load_v = [&]() -> bool {
      if (!v_pend) return true;
      const int vs = nv % kVStages;
      if (nv >= kVStages &&
          !__all_sync(0xffffffffu, mbar_wait(&bars.vempty[vs], ((nv / kVStages) - 1) & 1,
                                             &abort_sh, a.status, kWaitLimitNs)))
        return false;
      if (leader) {
        uint8_t* dst = dsm + Lay::kOffV + vs * Lay::kKVBytes;
        mbar_arrive_expect_tx(&bars.vfull[vs], Lay::kKVBytes);
        for (int c = 0; c < Lay::kChunks; ++c)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, &tmv, &bars.vfull[vs], c * 64,
                        (s ? pv_sub1 : pv_sub0) * kSubBlock, pv_kh, pv_b);
      }
      ++nv;
      v_pend = false;
      return true;
    };
    ok = publish_next();
    for (int k = 0; ok; ++k) {
      const Slot& S = slots[k % kSlots];
      if (S.item < 0) break;
      const int n_ent = S.n_ent, kh = S.h / group, b = S.b;
      // Q of the item, once the S products of the item that last used its stage have completed
      const int qs = nq % kQStages;
      if (nq >= kQStages &&
          !(ok = __all_sync(0xffffffffu, mbar_wait(&bars.q_empty[qs], ((nq / kQStages) - 1) & 1,
                                                   &abort_sh, a.status, kWaitLimitNs))))
        break;
      if (leader) {
        uint8_t* sq = dsm + Lay::kOffQ + qs * Lay::kQBytes;
        mbar_arrive_expect_tx(&bars.q_full[qs], Lay::kQBytes);
        for (int cc = 0; cc < Lay::kChunks; ++cc)
          for (int s = 0; s < 2; ++s)
            tma_load_4d(sq + cc * Lay::kChunkRowsQ + s * kBox, &tmq, &bars.q_full[qs], cc * 64,
                        s ? S.t1 : S.t0, S.h, b);
      }
      ++nq;
      const int n_steps = (n_ent + 1) / 2;
      for (int j = 0; j < n_steps; ++j) {
        const uint32_t e0 = S.ent[2 * j];
        const uint32_t e1 = (2 * j + 1 < n_ent) ? S.ent[2 * j + 1] : e0;
        const int sub0 = (int)(e0 & kSubMask), sub1 = (int)(e1 & kSubMask);
        // K of the step once the S product that last read its stage has completed
        const int ks = nk % kKStages;
        if (nk >= kKStages &&
            !(ok = __all_sync(0xffffffffu, mbar_wait(&bars.kempty[ks], ((nk / kKStages) - 1) & 1,
                                                     &abort_sh, a.status, kWaitLimitNs))))
          break;
        if (leader) {
          uint8_t* dst = dsm + Lay::kOffK + ks * Lay::kKVBytes;
          mbar_arrive_expect_tx(&bars.kfull[ks], Lay::kKVBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(dst + c * Lay::kChunkRowsKV + s * kBox, &tmk, &bars.kfull[ks], c * 64,
                          (s ? sub1 : sub0) * kSubBlock, kh, b);
        }
        ++nk;
        // V of the previous step (its product is issued after this step's S)
        if (!(ok = load_v())) break;
        v_pend = true;
        pv_sub0 = sub0;
        pv_sub1 = sub1;
        pv_kh = kh;
        pv_b = b;
        // the next item's list, while this one runs
        if (j == 0 && !ended && !(ok = publish_next())) break;
      }
    }
    if (ok) ok = load_v();
    if (leader) {
      if (!ok) raise_timeout(&abort_sh, a.status);
      // Drain: every copy issued above lands before the CTA exits (the last
      // copy into each stage; earlier ones completed before it was reused).
      volatile int no_abort = 0;
      for (int s = 0; s < kKStages; ++s) {
        const int c = nk - 1 - ((nk - 1 - s) % kKStages + kKStages) % kKStages;  // last copy into s
        if (c >= 0 && c % kKStages == s &&
            !mbar_wait(&bars.kfull[s], (c / kKStages) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
      }
      for (int s = 0; s < kVStages; ++s) {
        const int c = nv - 1 - ((nv - 1 - s) % kVStages + kVStages) % kVStages;
        if (c >= 0 && c % kVStages == s &&
            !mbar_wait(&bars.vfull[s], (c / kVStages) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
      }
      for (int s = 0; s < kQStages; ++s) {
        const int c = nq - 1 - ((nq - 1 - s) % kQStages + kQStages) % kQStages;
        if (c >= 0 && c % kQStages == s &&
            !mbar_wait(&bars.q_full[s], (c / kQStages) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
      }
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
    bool ok = true;
    int n = 0;  // steps whose S product was issued
    int t = 0;  // items
    // the step whose PV products are still to be issued
    bool pend = false, pend_first = false, pend_last = false;
    int pend_step = 0, pend_item = 0;
    // O_g += P_g V_g of the pending step m for both groups (keys 64 g .. 64 g + 63)
    auto issue_pv = [&]() -> bool {
      const int m = pend_step;
      const int vs = m % kVStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.vfull[vs], (m / kVStages) & 1, &abort_sh,
                                             a.status, kWaitLimitNs)))
        return false;
      // the first product of an item overwrites O: the previous epilogue must have read it
      if (pend_first && pend_item > 0 &&
          !__all_sync(0xffffffffu, mbar_wait(&bars.o_empty, (pend_item - 1) & 1, &abort_sh,
                                             a.status, kWaitLimitNs)))
        return false;
      const uint64_t dvs = dv + (uint64_t)((vs * Lay::kKVBytes) >> 4);
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.p_ready[g][m & 1], (m >> 1) & 1, &abort_sh,
                                               a.status, kWaitLimitNs)))
          return false;
        tc_fence_after();
        const uint32_t pcol = tmem + kColS + 128u * (uint32_t)(m & 1) + 64u * g;
        const uint32_t ocol = tmem + kColO + 128u * g;
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          // keys [64 g + 16 kq, +16): V rows of the stage (128 bytes each); P
          // elements packed in the group's columns [8 kq, 8 kq + 8)
          const int kk = 4 * g + kq;
          if (leader)
            mma_bf16_ts(ocol, pcol + 8 * kq, dvs + (uint64_t)((kk * 16 * 128) >> 4), idPV,
                        (pend_first && kq == 0) ? 0u : 1u);
        }
        if (leader) tc_commit(&bars.pv_done[g][m & 1]);
      }
      if (leader) {
        tc_commit(&bars.vempty[vs]);
        if (pend_last) tc_commit(&bars.o_full);
      }
      pend = false;
      return true;
    };
    for (int k = 0; ok; ++k) {
      const int slot = k % kSlots;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.list_full[slot], (k / kSlots) & 1,
                                                   &abort_sh, a.status, kWaitLimitNs))))
        break;
      const Slot& S = slots[slot];
      const int item_valid = S.item >= 0;
      const int n_steps = (S.n_ent + 1) / 2;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.list_empty[slot]);  // the slot's header was all it needed
      if (!item_valid) break;
      const int qs = t % kQStages;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.q_full[qs], (t / kQStages) & 1,
                                                   &abort_sh, a.status, kWaitLimitNs))))
        break;
      const uint64_t dqs = dq + (uint64_t)((qs * Lay::kQBytes) >> 4);
      for (int j = 0; j < n_steps; ++j) {
        // S(n) into buffer n % 2: its previous content S(n - 2) has been read
        // by both groups (their weights for step n - 2 were awaited before the
        // PV products of n - 2, issued ahead of this product)
        const int ks = n % kKStages;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars.kfull[ks], (n / kKStages) & 1,
                                                     &abort_sh, a.status, kWaitLimitNs))))
          break;
        tc_fence_after();
        const uint64_t dks = dk + (uint64_t)((ks * Lay::kKVBytes) >> 4);
        const uint32_t scol = tmem + kColS + 128u * (uint32_t)(n & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 d-columns: chunk kk / 4, 32 bytes (kk % 4) inside the swizzle atom
          const uint64_t offq = (uint64_t)(((kk / 4) * Lay::kChunkRowsQ + (kk % 4) * 32) >> 4);
          const uint64_t offk = (uint64_t)(((kk / 4) * Lay::kChunkRowsKV + (kk % 4) * 32) >> 4);
          if (leader) mma_bf16_ss(scol, dqs + offq, dks + offk, idS, kk > 0 ? 1u : 0u);
        }
        if (leader) {
          tc_commit(&bars.kempty[ks]);
          tc_commit(&bars.s_full[n & 1]);
          if (j == n_steps - 1) tc_commit(&bars.q_empty[qs]);
        }
        // then the PV products of the previous step
        if (pend && !(ok = issue_pv())) break;
        pend = true;
        pend_step = n;
        pend_first = j == 0;
        pend_last = j == n_steps - 1;
        pend_item = t;
        ++n;
      }
      ++t;
      // the item's last products go out now, not behind the next item's first
      // S product (which waits for that item's Q and K): the epilogue starts as
      // soon as the softmax has written the last weights
      if (ok && pend && !(ok = issue_pv())) break;
    }
    if (ok && pend) ok = issue_pv();
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
    const int sw = warp - kSoftWarp0;  // 0..7
    const int grp = sw / 4;            // 0: keys 0..63 of every step, 1: keys 64..127
    const int quad = warp & 3;         // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t ocol_own = trow + kColO + 128u * grp;
    const uint32_t ocol_oth = trow + kColO + 128u * (1 - grp);
    uint8_t* ostage = dsm + Lay::kOffO + sw * kOBoxBytes;
    const float sl2 = a.scale_log2;
    int n = 0;  // steps so far
    uint32_t xuses = 0;
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
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[n & 1], (n >> 1) & 1, &abort_sh,
                                               a.status, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        // this group's sub-block of the step (the padding of an odd list keeps nothing)
        const uint32_t e = grp == 0 ? (uint32_t)S.ent[2 * j]
                                    : ((2 * j + 1 < n_ent) ? (uint32_t)S.ent[2 * j + 1] : 0u);
        // (keep is uniform over a warp: its 32 rows lie in one query block)
        const bool keep = (e >> (kKeepShift + half)) & 1u;
        const uint32_t scol = trow + kColS + 128u * (uint32_t)(n & 1) + 64u * grp;
        uint32_t pw[32];
        if (keep) {
          // S in two 32-column chunks: the second loads while the first is
          // turned into weights
          uint32_t r[64];
          tmem_ld32(scol + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_wait_ld();
          tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          const uint64_t sl2x2 = pack2(sl2, sl2);
          float rsa = 0.f, rsb = 0.f;  // row sums of the rounded weights (low, high halves)
          uint64_t rx2 = pack2(0.f, 0.f);
          // (warp-uniform: a warp's rows share their keep bits, so either all
          // or none of them have kept a block of this item yet)
          const bool first = __any_sync(0xffffffffu, m == -INFINITY);
          float mt;
          if (first) {
            tmem_wait_ld();
            mt = fmaxf(max32(r), max32(r + 32)) * sl2;
          } else {
            // weights against the current reference while the tile maximum is
            // found alongside; they stand unless the maximum grew by more than 8
            const uint64_t nmx2 = pack2(-m, -m);
            weights32<kLse>(r, sl2x2, nmx2, pw, rsa, rsb, rx2);
            const float m0 = max32(r);
            tmem_st16(scol, *reinterpret_cast<uint32_t(*)[16]>(&pw[0]));
            tmem_wait_ld();
            weights32<kLse>(r + 32, sl2x2, nmx2, pw + 16, rsa, rsb, rx2);
            mt = fmaxf(m0, max32(r + 32)) * sl2;
          }
          const bool raise = mt > m + kRaiseLog2;
          if (first || __any_sync(0xffffffffu, raise)) {
            // O holds this group's products of the item's earlier steps; rows
            // that kept nothing yet (m = -inf) hold zeros and need no rescale
            if (j > 0 && __any_sync(0xffffffffu, raise && m != -INFINITY)) {
              // the product of step n - 1 completes before O is touched (the
              // barrier of steps of that parity: its phase n - 3 arrived before
              // S(n - 1)'s, which this group has seen, so the parity is exact)
              const int pm = n - 1;
              ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done[grp][pm & 1], (pm >> 1) & 1,
                                                     &abort_sh, a.status, kWaitLimitNs));
              if (!ok) break;
              tc_fence_after();
              const float alpha = (raise && m != -INFINITY) ? ex2_approx(m - mt) : 1.0f;
#pragma unroll 1
              for (int c = 0; c < D / 16; ++c) {
                uint32_t ov[16];
                tmem_ld16(ocol_own + c * 16, ov);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 16; ++x)
                  ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
                tmem_st16(ocol_own + c * 16, ov);
              }
              l *= alpha;
              lx *= alpha;
            }
            if (raise) m = mt;
            // the weights against the (new) reference
            const uint64_t nmx2 = pack2(-m, -m);
            rsa = rsb = 0.f;
            rx2 = pack2(0.f, 0.f);
            weights32<kLse>(r, sl2x2, nmx2, pw, rsa, rsb, rx2);
            weights32<kLse>(r + 32, sl2x2, nmx2, pw + 16, rsa, rsb, rx2);
            tmem_wait_st();  // an earlier store of the first chunk lands before this one
            tmem_st16(scol, *reinterpret_cast<uint32_t(*)[16]>(&pw[0]));
          }
          const float2 b2 = unpack2(rx2);
          l += rsa + rsb;
          lx += b2.x + b2.y;
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) pw[x] = 0u;
          tmem_st16(scol, *reinterpret_cast<uint32_t(*)[16]>(&pw[0]));
        }
        tmem_st16(scol + 16, *reinterpret_cast<uint32_t(*)[16]>(&pw[16]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_ready[grp][n & 1]);
      }
      if (!ok) break;
      // --------------------------------------------------------- epilogue
      // every product of the item has completed; the groups swap their row
      // maxima and sums, then each merges and writes half of O's columns
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bars.o_full, k & 1, &abort_sh, a.status, kWaitLimitNs));
      if (!ok) break;
      xm[grp][row] = m;
      xl[grp][row] = l;
      xlx[grp][row] = lx;
      ok = __all_sync(0xffffffffu, group_sync(&bars.xch, xuses, &abort_sh, a.status, kWaitLimitNs));
      if (!ok) break;
      const float m2 = xm[1 - grp][row], l2 = xl[1 - grp][row], lx2 = xlx[1 - grp][row];
      const float mf = fmaxf(m, m2);
      const float a_own = m != -INFINITY ? ex2_approx(m - mf) : 0.f;
      const float a_oth = m2 != -INFINITY ? ex2_approx(m2 - mf) : 0.f;
      const float lt = l * a_own + l2 * a_oth;
      const float inv = lt > 0.f ? 1.0f / lt : 0.f;
      const float s_own = a_own * inv, s_oth = a_oth * inv;
      // O / l as bf16, 32 columns at a time through this warp's staging box
      // (row `lane` holds its 64 bytes as four 16-byte chunks, chunk x at
      // x ^ ((lane / 2) % 4): the 64-byte swizzle), then one tensor store per
      // box; rows past L are clipped by the store
      const int tok0 = tok - lane;  // first token of this warp's 32 rows
#pragma unroll 1
      for (int c = grp * (D / 64); c < (grp + 1) * (D / 64); ++c) {
        uint32_t ov[32], ow[32];
        tmem_ld32(ocol_own + c * 32, ov);
        tmem_ld32(ocol_oth + c * 32, ow);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float o0 = __uint_as_float(ov[2 * x]) * s_own + __uint_as_float(ow[2 * x]) * s_oth;
          const float o1 =
              __uint_as_float(ov[2 * x + 1]) * s_own + __uint_as_float(ow[2 * x + 1]) * s_oth;
          __nv_bfloat162 v = __floats2bfloat162_rn(o0, o1);
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
      if (lane == 0) {
        mbar_arrive(&bars.o_empty);
        mbar_arrive(&bars.list_empty[slot]);
      }
      if (kLse && grp == 0 && a.lse && tok < a.L) {
        const float lxt = lx * a_own + lx2 * a_oth;
        a.lse[((int64_t)b * a.H + h) * a.L + tok] =
            lxt > 0.f ? (mf + log2f(lxt)) * 0.69314718055994531f : -INFINITY;
      }
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
    // this CTA takes no more items; the last one out checks the counter and
    // resets it for a later launch
    __threadfence();
    if (atomicAdd(&g_sched[sched_slot].finished, 1u) == gridDim.x - 1) {
      const unsigned taken = atomicExch(&g_sched[sched_slot].next, 0u);
      if (!(*(volatile int*)a.status & kDevTimeout) && taken != (unsigned)n_items + gridDim.x)
        atomicOr(a.status, kDevOverlap);
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
  // persistent CTAs, one per SM
  const int64_t n_items = (int64_t)a.B * a.H * ((a.L + kBM - 1) / kBM);
  const int64_t cap = (int64_t)g_num_sms[dev];
  const int grid = (int)(n_items < cap ? n_items : cap);
  if (a.d == 128)
    return a.lse ? launch_tc<128, true>(a, tq, tk, tv, to, st, grid, dev)
                 : launch_tc<128, false>(a, tq, tk, tv, to, st, grid, dev);
  return a.lse ? launch_tc<64, true>(a, tq, tk, tv, to, st, grid, dev)
               : launch_tc<64, false>(a, tq, tk, tv, to, st, grid, dev);
}

}  // namespace sdl
