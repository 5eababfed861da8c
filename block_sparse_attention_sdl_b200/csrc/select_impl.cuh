// Device code of the mask selection (radix select over the block scores),
// shared by the per-phase kernels of select.cu and the fused anchor kernel of
// anchor.cu.  See select.cu for the method.
#pragma once
#include <math.h>

#include "internal.cuh"

namespace sdl {
namespace selimpl {
namespace {  // internal linkage in every translation unit that includes this


constexpr int kBins = 2048;
constexpr int kPasses = 3;
__constant__ int kShift[kPasses] = {21, 10, 0};
__constant__ int kWidth[kPasses] = {11, 11, 10};
constexpr int kThreads = 256;

// Shared-memory histogram increment aggregated over the lanes of a warp that
// hit the same bin (block scores of one workload often share their top bits,
// which would otherwise serialise the atomics on one address).
__device__ __forceinline__ void hist_add(int* sh, int bin, bool active) {
  const unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, bin);
  const int leader = __ffs(peers) - 1;
  if ((int)(threadIdx.x % 32) == leader) atomicAdd(&sh[bin], __popc(peers));
}

struct SelWs {
  int* hist;      // [kPasses][B][kBins]
  int* gt;        // [R] off-diagonal scores above the threshold, per row
  int* eq;        // [R] off-diagonal scores equal to the threshold, per row
  int* take;      // [R] ties this row keeps
  uint32_t* tau;  // [B] threshold bit pattern (0xFFFFFFFF: no free picks)
  uint32_t* krem; // [B] threshold ties to keep (the chunked count and finish)
  int2* agg;      // [R] per row chunk: (ties, kept without ties) (chunked count)
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

SelWs carve(void* ws, int B, int R) {
  char* p = static_cast<char*>(ws);
  SelWs w;
  w.hist = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * (size_t)kPasses * B * kBins);
  w.gt = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * (size_t)R);
  w.eq = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * (size_t)R);
  w.take = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * (size_t)R);
  w.tau = reinterpret_cast<uint32_t*>(p);
  p += align256(sizeof(uint32_t) * (size_t)B);
  w.krem = reinterpret_cast<uint32_t*>(p);
  p += align256(sizeof(uint32_t) * (size_t)B);
  w.agg = reinterpret_cast<int2*>(p);
  return w;
}

// Bytes carve() lays out for B batch elements and R rows in total.
__host__ inline size_t carve_bytes(int B, size_t R) {
  return align256(sizeof(int) * (size_t)kPasses * B * kBins) + 3 * align256(sizeof(int) * R) +
         2 * align256(sizeof(uint32_t) * (size_t)B) + align256(sizeof(int2) * R);
}

// Block-wide: walk the histograms of passes [0, npass) of batch element b and
// return the digit prefix of the k-th largest key and how many of the keys
// sharing that prefix still have to be taken.  All threads of the block get
// the result.  Requires blockDim.x == kThreads.
//
// Every thread compares against its own copy of the prefix and the count
// left; the one thread whose bins hold the k-th key publishes the new values
// in shared memory, and all threads take them only after the next barrier.
// (Reading the shared count in the same barrier interval as its update let a
// late thread see the updated count, match one of its own bins as well and
// corrupt the prefix.)
__device__ void resolve(const int* hist, int B, int b, int npass, uint32_t kfree,
                        uint32_t* prefix_out, uint32_t* krem_out) {
  __shared__ uint32_t s_prefix, s_krem;
  __shared__ int s_warp[kThreads / 32];
  uint32_t prefix = 0, krem = kfree;
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_krem = kfree;
  }
  __syncthreads();
  for (int p = 0; p < npass; ++p) {
    const int nbin = 1 << kWidth[p];
    const int per = nbin / kThreads;  // 8 or 4 bins per thread
    const int* hb = hist + ((size_t)p * B + b) * kBins;
    // thread t owns bins [nbin - per*(t+1), nbin - per*t): thread 0 the top ones
    const int hi = nbin - per * threadIdx.x;
    int cnt[8];
    int local = 0;
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      cnt[x] = x < per ? hb[hi - 1 - x] : 0;
      local += cnt[x];
    }
    // exclusive scan of `local` over threads in order
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int incl = local;
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += s_warp[w];
    uint32_t above = (uint32_t)(wbase + incl - local);
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      if (x >= per) break;
      uint32_t c = (uint32_t)cnt[x];
      if (above < krem && above + c >= krem) {
        s_prefix = prefix | (uint32_t)(hi - 1 - x) << kShift[p];
        s_krem = krem - above;
      }
      above += c;
    }
    __syncthreads();
    prefix = s_prefix;
    krem = s_krem;
  }
  *prefix_out = prefix;
  *krem_out = krem;
  __syncthreads();  // the shared values may be rewritten by the block's next call
}


// Block (cx of ncx chunks, batch element b): histogram of digit `pass` over the
// off-diagonal scores of b whose higher digits match the resolved prefix.
// Requires blockDim.x == kThreads.
__device__ __forceinline__ void hist_body(const float* __restrict__ scores, int B, int H, int nb,
                                          uint32_t kfree, int pass, SelWs ws, int cx, int ncx,
                                          int b) {
  __shared__ int sh[kBins];
  if (kfree == 0) return;
  uint32_t prefix = 0, krem = kfree;
  if (pass > 0) resolve(ws.hist, B, b, pass, kfree, &prefix, &krem);
  for (int x = threadIdx.x; x < kBins; x += kThreads) sh[x] = 0;
  __syncthreads();
  const int shift = kShift[pass];
  const uint32_t dmask = (1u << kWidth[pass]) - 1u;
  const int hs = shift + kWidth[pass];  // bits at and above hs are fixed by the prefix
  const uint32_t want = hs >= 32 ? 0u : (prefix >> hs);
  const int64_t per_b = (int64_t)H * nb * nb;
  const float* base = scores + (int64_t)b * per_b;
  // 16-byte loads only when every batch element's slice starts 16-byte aligned
  const int64_t n4 = (per_b % 4 == 0) ? per_b / 4 : 0;
  // whole warps iterate together so the lane-aggregated increments stay convergent
  const int64_t n4_round = (n4 + kThreads - 1) / kThreads * kThreads;
  const bool narrow = per_b <= 0x7fffffff;  // 32-bit index arithmetic suffices
  for (int64_t x = (int64_t)cx * kThreads + threadIdx.x; x < n4_round;
       x += (int64_t)ncx * kThreads) {
    float vals[4] = {0.f, 0.f, 0.f, 0.f};
    const bool in = x < n4;
    int i = 0, j = 0;  // the first element's query block and key block
    if (in) {
      float4 v = __ldg(reinterpret_cast<const float4*>(base) + x);
      vals[0] = v.x;
      vals[1] = v.y;
      vals[2] = v.z;
      vals[3] = v.w;
      if (narrow) {
        const uint32_t e = 4u * (uint32_t)x, r = e / (uint32_t)nb;
        j = (int)(e - r * (uint32_t)nb);
        i = (int)(r % (uint32_t)nb);
      } else {
        const int64_t e = 4 * x, r = e / nb;
        j = (int)(e - r * nb);
        i = (int)(r % nb);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t key = __float_as_uint(vals[u]);
      const bool take = in && i != j && (hs >= 32 || (key >> hs) == want);
      hist_add(sh, (int)((key >> shift) & dmask), take);
      if (++j == nb) {  // the next element starts the next row
        j = 0;
        i = i + 1 == nb ? 0 : i + 1;
      }
    }
  }
  const int64_t tail0 = n4 * 4;
  const int64_t tail_round = tail0 + (per_b - tail0 + kThreads - 1) / kThreads * kThreads;
  for (int64_t e = tail0 + (int64_t)cx * kThreads + threadIdx.x; e < tail_round;
       e += (int64_t)ncx * kThreads) {
    const bool in = e < per_b;
    uint32_t key = 0;
    int i = 0, j = 0;
    if (in) {
      j = (int)(e % nb);
      i = (int)((e / nb) % nb);
      key = __float_as_uint(base[e]);
    }
    const bool take = in && i != j && (hs >= 32 || (key >> hs) == want);
    hist_add(sh, (int)((key >> shift) & dmask), take);
  }
  __syncthreads();
  int* gh = ws.hist + ((size_t)pass * B + b) * kBins;
  for (int x = threadIdx.x; x <= (int)dmask; x += kThreads)
    if (sh[x]) atomicAdd(&gh[x], sh[x]);
}

// Block (cx of ncx row chunks, batch element b); one warp per query-block row.
__device__ __forceinline__ void count_body(const float* __restrict__ scores, int B, int H, int nb,
                                           uint32_t kfree, SelWs ws, int cx, int ncx, int b) {
  uint32_t tau = 0xFFFFFFFFu, krem = 0;
  if (kfree > 0) resolve(ws.hist, B, b, kPasses, kfree, &tau, &krem);
  if (cx == 0 && threadIdx.x == 0) ws.tau[b] = tau;
  const int lane = threadIdx.x % 32;
  const int rows = H * nb;
  for (int r = cx * (kThreads / 32) + threadIdx.x / 32; r < rows;
       r += ncx * (kThreads / 32)) {
    const int i = r % nb;
    const int64_t row = (int64_t)b * rows + r;
    const float* pr = scores + row * nb;
    int gt = 0, eq = 0;
    for (int j = lane; j < nb; j += 32) {
      if (j == i) continue;
      uint32_t key = __float_as_uint(__ldg(pr + j));
      gt += key > tau && tau != 0xFFFFFFFFu;
      eq += key == tau;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
      ws.gt[row] = gt;
      ws.eq[row] = eq;
    }
  }
}

// Exclusive prefix of v over the threads of the block in thread order; `total`
// gets the block sum.  Every thread of the block must call it.
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nwarp = blockDim.x / 32;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarp ? s_warp[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    s_warp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int excl = (warp ? s_warp[warp - 1] : 0) + incl - v;
  total = s_warp[31];
  __syncthreads();  // s_warp may be reused
  return excl;
}

// One block (any multiple of 32 threads up to 1024): per batch element, the
// ties are handed out to rows in flat order (the tie-break), then the kept
// counts are scanned into row_ptr.  With `offs` (heads split over ranks;
// [B][2]: keys above the threshold over all ranks, threshold ties held by lower
// ranks) the tie quota and its start come from there instead of from this
// call's rows alone.
__device__ __forceinline__ void scan_body(int B, int H, int nb, uint32_t kfree, SelWs ws,
                                          int32_t* __restrict__ row_ptr,
                                          const int64_t* __restrict__ offs) {
  constexpr int R = 8;  // consecutive rows per thread and chunk
  __shared__ int s_warp[32];
  const int rows = H * nb;
  const int nthr = blockDim.x;
  int cnt_carry = 0;  // kept blocks of all earlier rows (the same in every thread)
  for (int b = 0; b < B; ++b) {
    // the ties each row takes: the threshold's remaining count, by flat index
    uint32_t krem = 0;
    {
      // ties to take = kfree - (number of scores above the threshold in batch b)
      int g = 0;
      for (int r = threadIdx.x; r < rows; r += nthr) g += ws.gt[(int64_t)b * rows + r];
      int total = 0;
      block_excl_scan(g, s_warp, total);
      krem = kfree - (uint32_t)(offs ? offs[2 * b] : (int64_t)total);
    }
    // ties held by lower ranks come first; more than the quota means none here
    const int64_t before0 = offs ? offs[2 * b + 1] : 0;
    int eq_carry = before0 > (int64_t)krem ? (int)krem : (int)before0;
    for (int r0 = 0; r0 < rows; r0 += nthr * R) {
      const int rb = r0 + (int)threadIdx.x * R;
      const int64_t base = (int64_t)b * rows + rb;
      int eqv[R], gtv[R], teq = 0;
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const bool in = rb + u < rows;
        eqv[u] = in ? ws.eq[base + u] : 0;
        gtv[u] = in ? ws.gt[base + u] : 0;
        teq += eqv[u];
      }
      int tot_eq = 0;
      int run = eq_carry + block_excl_scan(teq, s_warp, tot_eq);
      int cnt[R], take[R], tcnt = 0;
#pragma unroll
      for (int u = 0; u < R; ++u) {
        int t = (int)krem - run;
        t = t < 0 ? 0 : (t > eqv[u] ? eqv[u] : t);
        run += eqv[u];
        take[u] = t;
        cnt[u] = rb + u < rows ? gtv[u] + t + 1 : 0;
        tcnt += cnt[u];
      }
      int tot_cnt = 0;
      int pos = cnt_carry + block_excl_scan(tcnt, s_warp, tot_cnt);
#pragma unroll
      for (int u = 0; u < R; ++u) {
        if (rb + u < rows) {
          row_ptr[base + u] = pos;
          ws.take[base + u] = take[u];
        }
        pos += cnt[u];
      }
      eq_carry += tot_eq;
      cnt_carry += tot_cnt;
    }
  }
  if (threadIdx.x == 0) row_ptr[(int64_t)B * rows] = cnt_carry;
}

// Block (cx of ncx row chunks, batch element b); one warp per row writes its
// kept blocks in ascending j.
__device__ __forceinline__ void write_body(const float* __restrict__ scores, int B, int H, int nb,
                                           SelWs ws, const int32_t* __restrict__ row_ptr,
                                           int32_t* __restrict__ col_idx,
                                           uint8_t* __restrict__ mask, int cx, int ncx, int b) {
  const uint32_t tau = ws.tau[b];
  const int lane = threadIdx.x % 32;
  const int rows = H * nb;
  for (int r = cx * (kThreads / 32) + threadIdx.x / 32; r < rows;
       r += ncx * (kThreads / 32)) {
    const int i = r % nb;
    const int64_t row = (int64_t)b * rows + r;
    const float* pr = scores + row * nb;
    int pos = row_ptr[row];
    int ties_left = ws.take[row];
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      bool sel = false, tie = false;
      if (j < nb) {
        uint32_t key = __float_as_uint(__ldg(pr + j));
        if (j == i)
          sel = true;
        else if (tau != 0xFFFFFFFFu && key > tau)
          sel = true;
        else if (key == tau)
          tie = true;
      }
      const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
      if (tie) {
        int rank = __popc(tmask & ((1u << lane) - 1u));
        sel = rank < ties_left;
      }
      ties_left -= __popc(tmask);
      const uint32_t smask = __ballot_sync(0xffffffffu, sel);
      if (sel) col_idx[pos + __popc(smask & ((1u << lane) - 1u))] = j;
      if (mask && j < nb) mask[row * nb + j] = sel ? 1 : 0;
      pos += __popc(smask);
    }
  }
}

// ---- chunked variant (one launch; used by the fused anchor kernel)
//
// Pass 0 is histogrammed by the blocks that just wrote the scores (rows of one
// head), and the count, tie hand-out, row offsets and list writing run over
// contiguous chunks of rows: after the counts, a block takes the kept totals
// of every earlier chunk instead of waiting for one block's serial scan.  The
// results are those of hist/count/scan/write above (same keys, same rule).

// Pass-0 histogram of `nrows` rows of scores held in shared memory (`z`, row
// r at r * nb, query block i0 + r, of batch element b; off-diagonal scores),
// added into the pass-0 histogram of b.  Requires blockDim.x == kThreads;
// `sh`: kBins ints of shared memory apart from `z`.  A block barrier must
// separate the rows' writes from the call.
__device__ __forceinline__ void hist0_rows_body(const float* z, int nrows, int nb, int i0,
                                                uint32_t kfree, SelWs ws, int b, int* sh) {
  if (kfree == 0 || nrows <= 0) return;
  for (int x = threadIdx.x; x < kBins; x += kThreads) sh[x] = 0;
  __syncthreads();
  const int shift = kShift[0];
  const uint32_t dmask = (1u << kWidth[0]) - 1u;
  const int lane = threadIdx.x % 32;
  // one warp per row; every lane of a warp makes the same number of calls
  for (int r = (int)threadIdx.x / 32; r < nrows; r += kThreads / 32)
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const bool in = j < nb;
      const uint32_t key = in ? __float_as_uint(z[r * nb + j]) : 0u;
      hist_add(sh, (int)((key >> shift) & dmask), in && j != i0 + r);
    }
  __syncthreads();
  int* gh = ws.hist + (size_t)b * kBins;  // pass 0
  for (int x = threadIdx.x; x <= (int)dmask; x += kThreads)
    if (sh[x]) atomicAdd(&gh[x], sh[x]);
  __syncthreads();  // the bins may be reused by the block's next rows
}

// Rows [r0, r1) of chunk cx of ncx for H*nb rows per batch element.
__device__ __forceinline__ void chunk_rows(int rows, int cx, int ncx, int& r0, int& r1) {
  const int per = (rows + ncx - 1) / ncx;
  r0 = cx * per < rows ? cx * per : rows;
  r1 = r0 + per < rows ? r0 + per : rows;
}

// Block (chunk cx of ncx, batch element b), ncx <= H*nb: per-row counts of
// off-diagonal scores above and at the threshold, and the chunk's totals
// (ties, rows' kept entries without ties) in ws.agg[b * ncx + cx].  Chunk 0
// also stores the threshold and the ties to keep.
__device__ __forceinline__ void count_chunk_body(const float* __restrict__ scores, int B, int H,
                                                 int nb, uint32_t kfree, SelWs ws, int cx,
                                                 int ncx, int b) {
  __shared__ int s_eq, s_g1;
  uint32_t tau = 0xFFFFFFFFu, krem = 0;
  if (kfree > 0) resolve(ws.hist, B, b, kPasses, kfree, &tau, &krem);
  if (threadIdx.x == 0) {
    s_eq = 0;
    s_g1 = 0;
    if (cx == 0) {
      ws.tau[b] = tau;
      ws.krem[b] = krem;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x % 32;
  const int rows = H * nb;
  int r0, r1;
  chunk_rows(rows, cx, ncx, r0, r1);
  for (int r = r0 + (int)threadIdx.x / 32; r < r1; r += kThreads / 32) {
    const int i = r % nb;
    const int64_t row = (int64_t)b * rows + r;
    const float* pr = scores + row * nb;
    int gt = 0, eq = 0;
    for (int j = lane; j < nb; j += 32) {
      if (j == i) continue;
      const uint32_t key = __float_as_uint(__ldg(pr + j));
      gt += key > tau && tau != 0xFFFFFFFFu;
      eq += key == tau;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
      ws.gt[row] = gt;
      ws.eq[row] = eq;
      atomicAdd(&s_eq, eq);
      atomicAdd(&s_g1, gt + 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) ws.agg[(int64_t)b * ncx + cx] = make_int2(s_eq, s_g1);
}

// Block-wide sums of (x, y) over threads; every thread gets them.
__device__ __forceinline__ int2 block_sum2(int x, int y, int2* s_part) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nwarp = blockDim.x / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, o);
    y += __shfl_xor_sync(0xffffffffu, y, o);
  }
  if (lane == 0) s_part[warp] = make_int2(x, y);
  __syncthreads();
  int2 t = make_int2(0, 0);
  for (int w = 0; w < nwarp; ++w) {
    t.x += s_part[w].x;
    t.y += s_part[w].y;
  }
  __syncthreads();  // s_part may be reused
  return t;
}

// Block (chunk cx of ncx, batch element b), after every count_chunk_body:
// the chunk's rows' offsets into the lists and tie quotas (ties go to rows in
// flat order), then their kept blocks in ascending j (as write_body).  The
// chunk holding the last row of the last batch element writes the end offset.
__device__ __forceinline__ void finish_chunk_body(const float* __restrict__ scores, int B, int H,
                                                  int nb, SelWs ws, int32_t* __restrict__ row_ptr,
                                                  int32_t* __restrict__ col_idx, int cx, int ncx,
                                                  int b) {
  __shared__ int2 s_part[kThreads / 32];
  __shared__ int s_base;
  const int rows = H * nb;
  // kept entries of the earlier batch elements, then of the earlier chunks of b
  int base = 0, eq0 = 0;
  for (int bb = 0; bb <= b; ++bb) {
    const int nc = bb < b ? ncx : cx;
    int x = 0, y = 0;
    for (int c = threadIdx.x; c < nc; c += kThreads) {
      const int2 v = ws.agg[(int64_t)bb * ncx + c];
      x += v.x;
      y += v.y;
    }
    const int2 t = block_sum2(x, y, s_part);
    // ties go to the earliest rows: min(quota, ties seen) of them are kept
    const int kr = (int)ws.krem[bb];
    base += t.y + (t.x < kr ? t.x : kr);
    if (bb == b) eq0 = t.x;  // ties of the earlier chunks of b
  }
  int r0, r1;
  chunk_rows(rows, cx, ncx, r0, r1);
  const int krem = (int)ws.krem[b];
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int run_eq = eq0, pos = base;
    for (int c0 = r0; c0 < r1; c0 += 32) {
      const int r = c0 + lane;
      const int64_t row = (int64_t)b * rows + r;
      const int eqv = r < r1 ? ws.eq[row] : 0;
      const int gtv = r < r1 ? ws.gt[row] : 0;
      int ie = eqv;  // inclusive prefix of ties over the lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, ie, o);
        if (lane >= o) ie += u;
      }
      int t = krem - (run_eq + ie - eqv);
      t = t < 0 ? 0 : (t > eqv ? eqv : t);
      const int cnt = r < r1 ? gtv + t + 1 : 0;
      int ic = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, ic, o);
        if (lane >= o) ic += u;
      }
      if (r < r1) {
        row_ptr[row] = pos + ic - cnt;
        ws.take[row] = t;
      }
      run_eq += __shfl_sync(0xffffffffu, ie, 31);
      pos += __shfl_sync(0xffffffffu, ic, 31);
    }
    if (lane == 0) s_base = pos;
  }
  __syncthreads();
  if (threadIdx.x == 0 && b == B - 1 && r1 == rows && r0 < r1)
    row_ptr[(int64_t)B * rows] = s_base;
  // the chunk's lists (the offsets and quotas above are this block's writes)
  const uint32_t tau = ws.tau[b];
  const int lane = threadIdx.x % 32;
  for (int r = r0 + (int)threadIdx.x / 32; r < r1; r += kThreads / 32) {
    const int i = r % nb;
    const int64_t row = (int64_t)b * rows + r;
    const float* pr = scores + row * nb;
    int pos = row_ptr[row];
    int ties_left = ws.take[row];
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      bool sel = false, tie = false;
      if (j < nb) {
        const uint32_t key = __float_as_uint(__ldg(pr + j));
        if (j == i)
          sel = true;
        else if (tau != 0xFFFFFFFFu && key > tau)
          sel = true;
        else if (key == tau)
          tie = true;
      }
      const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
      if (tie) sel = __popc(tmask & ((1u << lane) - 1u)) < ties_left;
      ties_left -= __popc(tmask);
      const uint32_t smask = __ballot_sync(0xffffffffu, sel);
      if (sel) col_idx[pos + __popc(smask & ((1u << lane) - 1u))] = j;
      pos += __popc(smask);
    }
  }
}

// Block for batch element b: this call's keys above the threshold and equal
// to it (totals[2b], totals[2b+1]).
__device__ __forceinline__ void totals_body(int B, int H, int nb, SelWs ws,
                                            int64_t* __restrict__ totals, int b) {
  __shared__ unsigned long long s[2];
  if (threadIdx.x == 0) s[0] = s[1] = 0;
  __syncthreads();
  unsigned long long g = 0, e = 0;
  const int rows = H * nb;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) {
    g += ws.gt[(int64_t)b * rows + r];
    e += ws.eq[(int64_t)b * rows + r];
  }
  atomicAdd(&s[0], g);
  atomicAdd(&s[1], e);
  __syncthreads();
  if (threadIdx.x == 0) {
    totals[2 * b] = (int64_t)s[0];
    totals[2 * b + 1] = (int64_t)s[1];
  }
}

}  // namespace
}  // namespace selimpl
}  // namespace sdl
