// Key-major bf16 block-sparse attention on sm_100a tensor cores.
//
// The fused block-sparse kernel of the Step-dLLM abstract for 64-token blocks,
// laid out so that the 128-row dimension of the tensor-core tile runs over
// KEYS: every key a work item touches is one it keeps, so no MMA work is
// spent on blocks that only a neighbouring query block selected.
//
// Work item = one 64-row query tile (a 64-token query block, or half of a
// 128-token block) of one head, walking its kept key sub-blocks two at a time
// (128 keys per step).  Persistent CTAs take items in a static stride.
//
//   S^T = K Q^T     tcgen05.mma kind::f16, M = 128 keys, N = 64 queries, K = d;
//                   A = K tile, B = Q tile, both K-major in shared memory;
//                   fp32 accumulator in TMEM (two 64-column buffers).
//   softmax         one thread per key (its TMEM lane): p = exp2(s*c - m_q)
//                   with a per-query reference max m_q kept in shared memory;
//                   m_q is raised (and O^T, l rescaled) only when some logit
//                   exceeds it by more than 8 (log2 units), detected with one
//                   block-wide max per step.  P^T (bf16) goes to shared memory
//                   in the 128-byte-swizzled N-major operand layout.
//   O^T += V^T P^T  M = 128 = d, N = 64 queries, K = 128 keys; A = V tile read
//                   M-major, B = P^T N-major; TMEM accumulator (two buffers,
//                   one per item slot, so the epilogue of one item overlaps
//                   the next item's first products).
//   epilogue        per-query sums of the bf16 weights reduced across the 128
//                   key threads, O^T / l rounded to bf16 and stored, LSE.
//
// Warps: 0 K producer and 11 V producer (TMA, each its own ring so that K
// runs ahead of V), 1 TMEM allocator + MMA issuer, 2-9 softmax and epilogue in
// two warpgroups (each thread one key lane, one half of the query columns: two
// warps per scheduler hide each other's latencies), 10 item producer (kept
// list of the next item into shared memory and its Q tile by TMA, one item
// ahead).  Every wait is bounded.  The
// head dimension must be 128 (it is the M = 128 side of the O^T product).
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace sdl {
namespace {

constexpr int kRowsQ = 64;        // query rows per item
constexpr int kKeys = 128;        // keys per step (two 64-token sub-blocks)
constexpr int kKSt = 3;           // K ring depth (S runs ahead of PV)
constexpr int kVSt = 2;           // V ring depth
constexpr int kSlots = 2;         // item slots: list, Q tile, O^T accumulator
constexpr int kMaxSubKm = 1024;   // key sub-blocks per item (L <= 65536)
constexpr int kGroups = 2;        // softmax warpgroups, each owns 32 of the 64 query columns
constexpr int kCols = kRowsQ / kGroups;
constexpr int kSoftThreads = 128 * kGroups;
constexpr int kItemWarp = 2 + 4 * kGroups;      // warp index of the item producer
constexpr int kVWarp = kItemWarp + 1;            // warp index of the V producer
constexpr int kThreadsKm = 32 * (kVWarp + 1);
constexpr uint32_t kTmemColsKm = 256;
constexpr uint32_t kColS = 0;     // S^T buffers: columns 0 and 64
constexpr uint32_t kColO = 128;   // O^T buffers: columns 128 and 192
constexpr uint16_t kBadSub = 0xFFFFu;
constexpr int kBoxBytes = 64 * 128;  // one 64-row x 64-column bf16 box
constexpr float kRaise = 8.0f;       // log2 headroom before the reference max moves
constexpr int kPoly = 12;            // of each thread's 32 weights, how many take exp2_poly

template <int D>
struct KmLayout {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = kRowsQ * D * 2;
  static constexpr int kKVBytes = kKeys * D * 2;
  static constexpr int kPBytes = kKeys * kRowsQ * 2;
  static constexpr int kChunkQ = kRowsQ * 128;   // bytes per 64-column chunk of Q
  static constexpr int kChunkKV = kKeys * 128;   // bytes per 64-column chunk of K/V
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kSlots * kQBytes;
  static constexpr int kOffV = kOffK + kKSt * kKVBytes;
  static constexpr int kOffP = kOffV + kVSt * kKVBytes;
  static constexpr int kBytes = kOffP + kPBytes;
  static constexpr int kSmem = kBytes + 1024;  // + slack to align the base to 1024
};

struct KmBars {
  uint64_t list_full[kSlots], list_empty[kSlots];
  uint64_t q_full[kSlots], q_empty[kSlots];
  uint64_t k_full[kKSt], k_empty[kKSt];
  uint64_t v_full[kVSt], v_empty[kVSt];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t o_full[kSlots], o_empty[kSlots];
  uint64_t done;
  uint64_t soft[kGroups];  // barrier of each softmax warpgroup (128 threads)
};

struct KmSlot {
  int item;   // -1: no more work
  int n_sub;  // kept 64-token key sub-blocks
  int b, h, t0;
  uint16_t sub[kMaxSubKm];  // sub-block indices, kBadSub for rejected entries
};

struct KmShared {
  KmBars bars;
  KmSlot slot[kSlots];
  __align__(16) float nbias[kRowsQ];  // -m_q (log2 units): exponent reference per query
  __align__(16) float alpha[kRowsQ];  // rescale factors of a raise
  __align__(16) float lsum[kRowsQ];   // per-query inverse sums of the rounded weights
  __align__(16) float red[kGroups][4][kCols];  // cross-warp reduction buffer
  __align__(16) float emax[2][kGroups][4];     // per-warp step excess, by step parity
  uint32_t tmem_base;
  int abort_flag;
};

// 32 columns of this thread's TMEM lane as floats (warp-collective).
__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(r[q]);
}

__device__ __forceinline__ void km_raise_timeout(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicOr(status, kDevTimeout);
}

template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32], int lane) {
  // Reduce-scatter over the 32 lanes of a warp: v[32] holds one value per
  // column; after five butterfly levels lane L holds the reduction over all
  // lanes of column L.
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int m = 16 >> lvl;     // partner distance
    const int half = 16 >> lvl;  // values per side at this level
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < half) {
        const float keep = upper ? v[i + half] : v[i];
        const float send = upper ? v[i] : v[i + half];
        const float got = __shfl_xor_sync(0xffffffffu, send, m);
        v[i] = kMax ? fmaxf(keep, got) : keep + got;
      }
    }
  }
  return v[0];
}

template <int D, bool kLse>
__global__ void __launch_bounds__(kThreadsKm, 1)
    attn_km_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, AttnArgs a) {
  static_assert(D == 128, "the key-major kernel needs d = 128");
  using Lay = KmLayout<D>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                            ~(uintptr_t)1023);
  __shared__ KmShared sh;
  KmBars& bars = sh.bars;
  volatile int* abort_sh = &sh.abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_q64 = a.L / kRowsQ;
  const int n_items = a.B * a.H * n_q64;

  if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < kSlots; ++s) {
        mbar_init(&bars.list_full[s], 1);
        mbar_init(&bars.list_empty[s], 1 + kSoftThreads);
        mbar_init(&bars.q_full[s], 1);
        mbar_init(&bars.q_empty[s], 1);
        mbar_init(&bars.o_full[s], 1);
        mbar_init(&bars.o_empty[s], kSoftThreads);
      }
      for (int s = 0; s < kKSt; ++s) {
        mbar_init(&bars.k_full[s], 1);
        mbar_init(&bars.k_empty[s], 1);
      }
      for (int s = 0; s < kVSt; ++s) {
        mbar_init(&bars.v_full[s], 1);
        mbar_init(&bars.v_empty[s], 1);
      }
      mbar_init(&bars.s_full[0], 1);
      mbar_init(&bars.s_full[1], 1);
      mbar_init(&bars.p_full, kSoftThreads);
      mbar_init(&bars.pv_done, 1);
      mbar_init(&bars.done, 1);
      for (int gq = 0; gq < kGroups; ++gq) mbar_init(&bars.soft[gq], 128);
      sh.abort_flag = 0;
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(&sh.tmem_base, kTmemColsKm);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == kItemWarp) {
    // ======================================================= item producer
    int qiss0 = 0, qiss1 = 0;  // Q loads issued per slot
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = blockIdx.x + k * gridDim.x;  // static stride over items
      const bool have = item < n_items;
      const int slot = k % kSlots;
      if (k >= kSlots && lane == 0)
        ok = mbar_wait(&bars.list_empty[slot], ((k / kSlots) - 1) & 1, abort_sh, a.status,
                       kWaitLimitNs);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      KmSlot& S = sh.slot[slot];
      int n_sub = 0, b = 0, h = 0, t0 = 0;
      if (have) {
        b = item / (a.H * n_q64);
        h = (item / n_q64) % a.H;
        t0 = (item % n_q64) * kRowsQ;
        if (a.row_ptr == nullptr) {
          n_sub = a.L / kSubBlock;
          for (int e = lane; e < n_sub; e += 32) S.sub[e] = (uint16_t)e;
        } else {
          const int i = t0 / a.block;
          const int64_t r = ((int64_t)b * a.H + h) * a.nb + i;
          const int beg = a.row_ptr[r], end = a.row_ptr[r + 1];
          const int per = a.block / kSubBlock;  // 1 or 2
          int n = end - beg;
          if (n < 0 || n * per > kMaxSubKm) {
            if (lane == 0) atomicOr(a.status, kDevBadMask);
            n = n < 0 ? 0 : kMaxSubKm / per;
          }
          n_sub = n * per;
          for (int x = lane; x < n; x += 32) {
            const int j = a.col_idx[beg + x];
            bool bad = j < 0 || j >= a.nb;
            if (!bad && x > 0 && a.col_idx[beg + x - 1] >= j) bad = true;  // order / duplicate
            if (bad) atomicOr(a.status, kDevBadMask);
            for (int u = 0; u < per; ++u)
              S.sub[x * per + u] = bad ? kBadSub : (uint16_t)(j * per + u);
          }
        }
      }
      if (lane == 0) {
        S.item = have ? item : -1;
        S.n_sub = n_sub;
        S.b = b;
        S.h = h;
        S.t0 = t0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.list_full[slot]);
      if (!have) break;
      if (lane == 0 && n_sub > 0) {
        const int qiss = slot ? qiss1 : qiss0;
        if (qiss > 0)
          ok = mbar_wait(&bars.q_empty[slot], (qiss - 1) & 1, abort_sh, a.status, kWaitLimitNs);
        if (ok) {
          uint8_t* sq = dsm + Lay::kOffQ + slot * Lay::kQBytes;
          mbar_arrive_expect_tx(&bars.q_full[slot], Lay::kQBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            tma_load_4d(sq + c * Lay::kChunkQ, &tmq, &bars.q_full[slot], c * 64, t0, h, b);
          if (slot) ++qiss1; else ++qiss0;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      if (!ok) km_raise_timeout(abort_sh, a.status);
      volatile int no_abort = 0;
      if (qiss0 && !mbar_wait(&bars.q_full[0], (qiss0 - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
      if (qiss1 && !mbar_wait(&bars.q_full[1], (qiss1 - 1) & 1, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
    }
  } else if (warp == 0 || warp == kVWarp) {
    // ================================================= K and V producers
    // Warp 0 streams K tiles, warp kVWarp V tiles; each walks the items in
    // order and fills its own ring (step g uses slot g % depth).
    const bool isk = warp == 0;
    const int depth = isk ? kKSt : kVSt;
    uint64_t* full = isk ? bars.k_full : bars.v_full;
    uint64_t* empty = isk ? bars.k_empty : bars.v_empty;
    const CUtensorMap* tm = isk ? &tmk : &tmv;
    uint8_t* ring = dsm + (isk ? Lay::kOffK : Lay::kOffV);
    if (lane == 0) {
      int g = 0;  // global step
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kSlots;
        if (!(ok = mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, abort_sh, a.status,
                             kWaitLimitNs)))
          break;
        const KmSlot& S = sh.slot[slot];
        if (S.item < 0) break;
        const int n_sub = S.n_sub, b = S.b;
        const int kh = S.h / (a.H / a.Hkv);
        const int steps = (n_sub + 1) / 2;
        for (int j = 0; j < steps; ++j) {
          int sub0 = S.sub[2 * j];
          int sub1 = (2 * j + 1 < n_sub) ? S.sub[2 * j + 1] : sub0;
          if (sub0 == kBadSub) sub0 = 0;  // loaded but masked by the softmax
          if (sub1 == kBadSub) sub1 = sub0;
          const int rs = g % depth;
          if (g >= depth &&
              !(ok = mbar_wait(&empty[rs], ((g / depth) - 1) & 1, abort_sh, a.status,
                               kWaitLimitNs)))
            break;
          uint8_t* dst = ring + rs * Lay::kKVBytes;
          mbar_arrive_expect_tx(&full[rs], Lay::kKVBytes);
          for (int c = 0; c < Lay::kChunks; ++c)
            for (int s = 0; s < 2; ++s)
              tma_load_4d(dst + c * Lay::kChunkKV + s * kBoxBytes, tm, &full[rs], c * 64,
                          (s ? sub1 : sub0) * kSubBlock, kh, b);
          ++g;
        }
      }
      if (!ok) km_raise_timeout(abort_sh, a.status);
      // Drain: every copy issued above lands before the CTA exits (only the
      // last ring-depth loads can still be in flight).
      volatile int no_abort = 0;
      for (int st = (g > depth ? g - depth : 0); st < g; ++st)
        if (!mbar_wait(&full[st % depth], (st / depth) & 1, &no_abort, nullptr, kWaitLimitNs))
          atomicOr(a.status, kDevTimeout);
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, kRowsQ, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, kRowsQ, true, true);
      const uint32_t q_base = smem_u32(dsm + Lay::kOffQ);
      const uint32_t k_base = smem_u32(dsm + Lay::kOffK);
      const uint32_t v_base = smem_u32(dsm + Lay::kOffV);
      const uint32_t p_base = smem_u32(dsm + Lay::kOffP);
      int quse0 = 0, quse1 = 0;  // Q tiles consumed per slot
      int ouse0 = 0, ouse1 = 0;  // O^T accumulations completed per slot
      bool ok = true;

      // Opens item ordinal k: waits for its list; returns its step count (0 for
      // an empty item) or -1 at the end of the schedule.
      auto open_item = [&](int k) -> int {
        const int slot = k % kSlots;
        if (!mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, abort_sh, a.status,
                       kWaitLimitNs)) {
          ok = false;
          return -1;
        }
        const KmSlot& S = sh.slot[slot];
        if (S.item < 0) return -1;
        return (S.n_sub + 1) / 2;
      };
      // Finds the next non-empty item at or after ordinal k (empty items are
      // released at once).  Returns its step count, or -1.
      auto next_item = [&](int& k) -> int {
        for (;;) {
          const int steps = open_item(k);
          if (steps != 0) return steps;
          mbar_arrive(&bars.list_empty[k % kSlots]);
          ++k;
        }
      };
      auto issue_s = [&](int g, int slot) -> bool {
        const int ks = g % kKSt;
        if (!mbar_wait(&bars.k_full[ks], (g / kKSt) & 1, abort_sh, a.status, kWaitLimitNs))
          return false;
        tc_fence_after();
        const uint32_t kb = k_base + ks * Lay::kKVBytes;
        const uint32_t qb = q_base + slot * Lay::kQBytes;
        const uint32_t dcol = tmem + kColS + 64u * (uint32_t)(g & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk % 4) * 32;
          const uint64_t ad = smem_desc_sw128(kb + (kk / 4) * Lay::kChunkKV + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(qb + (kk / 4) * Lay::kChunkQ + off, 16, 1024);
          mma_bf16_ss(dcol, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars.k_empty[ks]);
        tc_commit(&bars.s_full[g & 1]);
        return true;
      };

      int k = 0;
      int steps = next_item(k);
      int j = 0, g = 0;
      if (steps > 0) {
        int slot = k % kSlots;
        ok = mbar_wait(&bars.q_full[slot], (slot ? quse1 : quse0) & 1, abort_sh, a.status,
                       kWaitLimitNs);
        if (slot) ++quse1; else ++quse0;
        if (ok) ok = issue_s(0, slot);
        if (ok && steps == 1) tc_commit(&bars.q_empty[slot]);
        while (ok) {
          // look one step ahead, into the next item if this one ends here
          int k2 = k, j2 = j + 1, steps2 = steps;
          bool nxt = true;
          if (j2 == steps) {
            k2 = k + 1;
            j2 = 0;
            steps2 = next_item(k2);
            if (!ok) break;
            if (steps2 < 0) {
              nxt = false;
            } else {
              const int s2 = k2 % kSlots;
              if (!(ok = mbar_wait(&bars.q_full[s2], (s2 ? quse1 : quse0) & 1, abort_sh,
                                   a.status, kWaitLimitNs)))
                break;
              if (s2) ++quse1; else ++quse0;
            }
          }
          // Next S first if its K tile has landed (keeps the tensor pipe fed);
          // otherwise this step's O^T product goes first.
          bool s_issued = !nxt;
          if (nxt && mbar_test_wait(&bars.k_full[(g + 1) % kKSt], ((g + 1) / kKSt) & 1)) {
            if (!(ok = issue_s(g + 1, k2 % kSlots))) break;
            if (j2 == steps2 - 1) tc_commit(&bars.q_empty[k2 % kSlots]);
            s_issued = true;
          }
          // O^T += V^T P^T for the current step
          slot = k % kSlots;
          if (!(ok = mbar_wait(&bars.p_full, g & 1, abort_sh, a.status, kWaitLimitNs))) break;
          const int vs = g % kVSt;
          if (!(ok = mbar_wait(&bars.v_full[vs], (g / kVSt) & 1, abort_sh, a.status,
                               kWaitLimitNs)))
            break;
          const int ouse = slot ? ouse1 : ouse0;
          if (j == 0 && ouse > 0 &&
              !(ok = mbar_wait(&bars.o_empty[slot], (ouse - 1) & 1, abort_sh, a.status,
                               kWaitLimitNs)))
            break;
          tc_fence_after();
          const uint32_t vb = v_base + vs * Lay::kKVBytes;
          const uint32_t ocol = tmem + kColO + 64u * (uint32_t)slot;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(vb + kk * 16 * 128, Lay::kChunkKV, 1024);
            const uint64_t bd = smem_desc_sw128(p_base + kk * 16 * 128, Lay::kPBytes, 1024);
            mma_bf16_ss(ocol, ad, bd, idPV, (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bars.v_empty[vs]);
          tc_commit(&bars.pv_done);
          if (j == steps - 1) {
            tc_commit(&bars.o_full[slot]);
            if (slot) ++ouse1; else ++ouse0;
            mbar_arrive(&bars.list_empty[slot]);
          }
          if (!s_issued) {
            if (!(ok = issue_s(g + 1, k2 % kSlots))) break;
            if (j2 == steps2 - 1) tc_commit(&bars.q_empty[k2 % kSlots]);
          }
          if (!nxt) break;
          k = k2;
          j = j2;
          steps = steps2;
          ++g;
        }
      }
      if (!ok) km_raise_timeout(abort_sh, a.status);
      tc_commit(&bars.done);
      volatile int no_abort = 0;
      if (!mbar_wait(&bars.done, 0, &no_abort, nullptr, kWaitLimitNs))
        atomicOr(a.status, kDevTimeout);
    }
  } else {
    // ============================================================ softmax
    const int grp = (warp - 2) / 4;  // column half: queries [32 grp, 32 grp + 32)
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    const int t = quad * 32 + lane;  // key lane during a step, d row in the epilogue
    const int c0 = grp * kCols;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float c = a.scale_log2;
    uint8_t* pbase = dsm + Lay::kOffP;
    int ouse0 = 0, ouse1 = 0;  // O^T results consumed per slot
    uint32_t soft_uses = 0;
    int g = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % kSlots;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&bars.list_full[slot], (k / kSlots) & 1, abort_sh, a.status,
                                kWaitLimitNs));
      if (!ok) break;
      const KmSlot& S = sh.slot[slot];
      const int item = S.item;
      if (item < 0) break;
      const int n_sub = S.n_sub, b = S.b, h = S.h, t0 = S.t0;
      const int steps = (n_sub + 1) / 2;
      if (steps == 0) {
        // empty list (only from a rejected mask): zero output, -inf LSE
        __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                            (int64_t)(t0 + c0) * a.os[1] + h * a.os[2] + t;
        for (int q = 0; q < kCols; ++q) op[(int64_t)q * a.os[1]] = __float2bfloat16(0.f);
        if (a.lse && quad == 0) a.lse[((int64_t)b * a.H + h) * a.L + t0 + c0 + lane] = -INFINITY;
        mbar_arrive(&bars.list_empty[slot]);
        continue;
      }
      float lp[kCols];
      float lx[kCols];  // only used (and kept) when the LSE is requested
#pragma unroll
      for (int q = 0; q < kCols; ++q) lp[q] = lx[q] = 0.f;
      for (int j = 0; j < steps; ++j, ++g) {
        const int buf = g & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[buf], (g >> 1) & 1, abort_sh,
                                               a.status, kWaitLimitNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t scol = trow + kColS + 64u * (uint32_t)buf + (uint32_t)c0;
        float sv[kCols];
        tmem_ld32f(scol, sv);
        const int e = 2 * j + (t >> 6);
        const bool valid = e < n_sub && S.sub[e] != kBadSub;
        // Fast path (j > 0): weights against the current reference, computed
        // before the group learns whether any logit rose more than kRaise
        // above it; then one group barrier; the rare raise recomputes.
        bool slow = j == 0;
        if (!slow) {
          float ex = -INFINITY;
#pragma unroll
          for (int q = 0; q < kCols; q += 4) {
            const float4 nb4 = *reinterpret_cast<const float4*>(&sh.nbias[c0 + q]);
            sv[q] = valid ? fmaf(sv[q], c, nb4.x) : -INFINITY;
            sv[q + 1] = valid ? fmaf(sv[q + 1], c, nb4.y) : -INFINITY;
            sv[q + 2] = valid ? fmaf(sv[q + 2], c, nb4.z) : -INFINITY;
            sv[q + 3] = valid ? fmaf(sv[q + 3], c, nb4.w) : -INFINITY;
            ex = fmaxf(ex, fmaxf(fmaxf(sv[q], sv[q + 1]), fmaxf(sv[q + 2], sv[q + 3])));
          }
#pragma unroll
          for (int q = 0; q < kCols; ++q)
            sv[q] = q < kCols - kPoly ? ex2_approx(sv[q]) : exp2_poly(sv[q]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ex = fmaxf(ex, __shfl_xor_sync(0xffffffffu, ex, o));
          if (lane == 0) sh.emax[g & 1][grp][quad] = ex;
          if (!(ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs)))
            break;
          const float4 e4 = *reinterpret_cast<const float4*>(&sh.emax[g & 1][grp][0]);
          slow = fmaxf(fmaxf(e4.x, e4.y), fmaxf(e4.z, e4.w)) > kRaise;
        }
        if (slow) {
          // ---- raise the reference max (always at an item's first step).
          // Absolute logits a = s * c, re-read from TMEM (S^T(g) stays until
          // every softmax thread has released P(g)).
          tmem_ld32f(scol, sv);
#pragma unroll
          for (int q = 0; q < kCols; ++q) sv[q] = valid ? sv[q] * c : -INFINITY;
          const float mw = warp_reduce_scatter32<true>(sv, lane);
          sh.red[grp][quad][lane] = mw;
          if (!(ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs)))
            break;
          if (quad == 0) {
            const int q = c0 + lane;
            const float mt = fmaxf(fmaxf(sh.red[grp][0][lane], sh.red[grp][1][lane]),
                                   fmaxf(sh.red[grp][2][lane], sh.red[grp][3][lane]));
            if (j == 0) {
              sh.nbias[q] = mt == -INFINITY ? 0.f : -mt;
              sh.alpha[q] = 0.f;
            } else {
              const float mo = -sh.nbias[q];
              const float mn = fmaxf(mo, mt);
              sh.alpha[q] = ex2_approx(mo - mn);
              sh.nbias[q] = -mn;
            }
          }
          if (!(ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs)))
            break;
          if (j > 0) {
            // rescale this thread's partial sums and its row (d = t) of O^T
#pragma unroll
            for (int q = 0; q < kCols; ++q) lp[q] *= sh.alpha[c0 + q];
            if constexpr (kLse) {
#pragma unroll
              for (int q = 0; q < kCols; ++q) lx[q] *= sh.alpha[c0 + q];
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (g - 1) & 1, abort_sh,
                                                   a.status, kWaitLimitNs));
            if (!ok) break;
            tc_fence_after();
            uint32_t orow[kCols];
            const uint32_t oc = trow + kColO + 64u * (uint32_t)slot + (uint32_t)c0;
            tmem_ld32(oc, orow);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < kCols; ++q)
              orow[q] = __float_as_uint(__uint_as_float(orow[q]) * sh.alpha[c0 + q]);
            tmem_st32(oc, orow);
            tmem_wait_st();
          }
          tmem_ld32f(scol, sv);
#pragma unroll
          for (int q = 0; q < kCols; ++q) {
            const float x = valid ? fmaf(sv[q], c, sh.nbias[c0 + q]) : -INFINITY;
            sv[q] = q < kCols - kPoly ? ex2_approx(x) : exp2_poly(x);
          }
        }
        // ---- P^T row of this key: bf16 weights, sums of the rounded values
        uint32_t pw[kCols / 2];
#pragma unroll
        for (int q = 0; q < kCols; q += 2) {
          __nv_bfloat162 pk = __floats2bfloat162_rn(sv[q], sv[q + 1]);
          const uint32_t u = *reinterpret_cast<uint32_t*>(&pk);
          lp[q] += __uint_as_float(u << 16);
          lp[q + 1] += __uint_as_float(u & 0xFFFF0000u);
          if constexpr (kLse) {
            lx[q] += sv[q];
            lx[q + 1] += sv[q + 1];
          }
          pw[q / 2] = u;
        }
        // the single P^T buffer is free once the previous product finished
        if (g > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done, (g - 1) & 1, abort_sh, a.status,
                                                 kWaitLimitNs));
          if (!ok) break;
        }
        uint8_t* prow = pbase + t * 128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int chunk = grp * 4 + cc;  // 16-byte chunk of 8 queries
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (t & 7)) << 4)) =
              make_uint4(pw[4 * cc], pw[4 * cc + 1], pw[4 * cc + 2], pw[4 * cc + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars.p_full);
      }
      if (!ok) break;
      // ================================================== item epilogue
      {
        const float sw = warp_reduce_scatter32<false>(lp, lane);
        sh.red[grp][quad][lane] = sw;
        ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs);
        if (quad == 0) {
          const float l = (sh.red[grp][0][lane] + sh.red[grp][1][lane]) +
                          (sh.red[grp][2][lane] + sh.red[grp][3][lane]);
          sh.lsum[c0 + lane] = l > 0.f ? 1.0f / l : 0.f;  // inverse of the weight sum
        }
        if constexpr (kLse) {
          ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs) && ok;
          const float xw = warp_reduce_scatter32<false>(lx, lane);
          sh.red[grp][quad][lane] = xw;
          ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs) && ok;
          if (quad == 0) {
            const float lxs = (sh.red[grp][0][lane] + sh.red[grp][1][lane]) +
                              (sh.red[grp][2][lane] + sh.red[grp][3][lane]);
            a.lse[((int64_t)b * a.H + h) * a.L + t0 + c0 + lane] =
                lxs > 0.f ? (log2f(lxs) - sh.nbias[c0 + lane]) * 0.69314718055994531f
                          : -INFINITY;
          }
        }
        ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs) && ok;
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.o_full[slot], (slot ? ouse1 : ouse0) & 1,
                                             abort_sh, a.status, kWaitLimitNs));
      if (!ok) break;
      if (slot) ++ouse1; else ++ouse0;
      tc_fence_after();
      uint32_t orow[kCols];
      tmem_ld32(trow + kColO + 64u * (uint32_t)slot + (uint32_t)c0, orow);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars.o_empty[slot]);
      __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(a.o) + b * a.os[0] +
                          (int64_t)(t0 + c0) * a.os[1] + h * a.os[2] + t;
#pragma unroll
      for (int q = 0; q < kCols; ++q)
        op[(int64_t)q * a.os[1]] = __float2bfloat16_rn(__uint_as_float(orow[q]) * sh.lsum[c0 + q]);
      // lsum / red reuse by the next item
      if (!(ok = group_sync(&bars.soft[grp], soft_uses, abort_sh, a.status, kWaitLimitNs))) break;
      mbar_arrive(&bars.list_empty[slot]);
    }
    if (!ok) km_raise_timeout(abort_sh, a.status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemColsKm);
  }
}

int g_num_sms[64] = {0};

}  // namespace

template <int D, bool kLse>
static cudaError_t launch_km(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, cudaStream_t st, int grid) {
  using Lay = KmLayout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_km_kernel<D, kLse>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kSmem);
  if (e != cudaSuccess) return e;
  attn_km_kernel<D, kLse><<<grid, kThreadsKm, Lay::kSmem, st>>>(*tq, *tk, *tv, a);
  return cudaGetLastError();
}

cudaError_t launch_attn_km(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (g_num_sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int n_items = a.B * a.H * (a.L / kRowsQ);
  const int grid = n_items < g_num_sms[dev] ? n_items : g_num_sms[dev];
  if (a.d != 128) return cudaErrorInvalidValue;
  return a.lse ? launch_km<128, true>(a, tq, tk, tv, st, grid)
               : launch_km<128, false>(a, tq, tk, tv, st, grid);
}

}  // namespace sdl
