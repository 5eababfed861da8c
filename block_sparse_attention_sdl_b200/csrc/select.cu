// Mask selection for anchor steps: the head-adaptive global budget of the
// Step-dLLM abstract.  Per batch element the diagonal block of every query
// row is kept and the remaining budget goes to the largest off-diagonal block
// scores of all heads together, ties broken by the lower flat index.
//
// Exact k-th-largest search by radix select on the fp32 bit patterns (scores
// are softmax outputs, so non-negative, and their bit patterns order like the
// values): three digit passes of 11, 11 and 10 bits, each a shared-memory
// histogram per CTA merged into a global histogram with integer atomics.
// Every later kernel re-derives the threshold from the histograms, which is
// deterministic.  Then per-row counts, one scan for the tie quota of each row
// and the CSR offsets, and a warp-per-row compaction in ascending j.
#include <math.h>

#include "internal.cuh"

namespace sdl {
namespace {

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
  return w;
}

// Block-wide: walk the histograms of passes [0, npass) of batch element b and
// return the digit prefix of the k-th largest key and how many of the keys
// sharing that prefix still have to be taken.  All threads of the block get
// the result.  Requires blockDim.x == kThreads.
__device__ void resolve(const int* hist, int B, int b, int npass, uint32_t kfree,
                        uint32_t* prefix_out, uint32_t* krem_out) {
  __shared__ uint32_t s_prefix, s_krem;
  __shared__ int s_warp[kThreads / 32];
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
    for (int x = 0; x < per; ++x) {
      cnt[x] = hb[hi - 1 - x];
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
    const uint32_t krem = s_krem;
    uint32_t above = (uint32_t)(wbase + incl - local);
    for (int x = 0; x < per; ++x) {
      uint32_t c = (uint32_t)cnt[x];
      if (above < krem && above + c >= krem) {
        s_prefix |= (uint32_t)(hi - 1 - x) << kShift[p];
        s_krem = krem - above;
      }
      above += c;
    }
    __syncthreads();
  }
  *prefix_out = s_prefix;
  *krem_out = s_krem;
  __syncthreads();
}

__global__ void zero_kernel(int* p, size_t n) {
  for (size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x; x < n;
       x += (size_t)gridDim.x * blockDim.x)
    p[x] = 0;
}

// grid: (chunks, B).  Histogram of digit `pass` over the off-diagonal scores of
// batch element blockIdx.y whose higher digits match the resolved prefix.
__global__ void __launch_bounds__(kThreads) hist_kernel(const float* __restrict__ scores, int B,
                                                        int H, int nb, uint32_t kfree, int pass,
                                                        SelWs ws) {
  __shared__ int sh[kBins];
  const int b = blockIdx.y;
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
  for (int64_t x = (int64_t)blockIdx.x * kThreads + threadIdx.x; x < n4_round;
       x += (int64_t)gridDim.x * kThreads) {
    float vals[4] = {0.f, 0.f, 0.f, 0.f};
    const bool in = x < n4;
    if (in) {
      float4 v = __ldg(reinterpret_cast<const float4*>(base) + x);
      vals[0] = v.x;
      vals[1] = v.y;
      vals[2] = v.z;
      vals[3] = v.w;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = 4 * x + u;
      const int j = (int)(e % nb);
      const int i = (int)((e / nb) % nb);
      const uint32_t key = __float_as_uint(vals[u]);
      const bool take = in && i != j && (hs >= 32 || (key >> hs) == want);
      hist_add(sh, (int)((key >> shift) & dmask), take);
    }
  }
  const int64_t tail0 = n4 * 4;
  const int64_t tail_round = tail0 + (per_b - tail0 + kThreads - 1) / kThreads * kThreads;
  for (int64_t e = tail0 + (int64_t)blockIdx.x * kThreads + threadIdx.x; e < tail_round;
       e += (int64_t)gridDim.x * kThreads) {
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

// grid: (row chunks, B); one warp per query-block row.
__global__ void __launch_bounds__(kThreads) count_kernel(const float* __restrict__ scores, int B,
                                                         int H, int nb, uint32_t kfree,
                                                         SelWs ws) {
  const int b = blockIdx.y;
  uint32_t tau = 0xFFFFFFFFu, krem = 0;
  if (kfree > 0) resolve(ws.hist, B, b, kPasses, kfree, &tau, &krem);
  if (blockIdx.x == 0 && threadIdx.x == 0) ws.tau[b] = tau;
  const int lane = threadIdx.x % 32;
  const int rows = H * nb;
  for (int r = blockIdx.x * (kThreads / 32) + threadIdx.x / 32; r < rows;
       r += gridDim.x * (kThreads / 32)) {
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

// One CTA of 1024 threads: per batch element, the ties are handed out to rows
// in flat order (the tie-break), then the kept counts are scanned into row_ptr.
// With `offs` (heads split over ranks; [B][2]: keys above the threshold over
// all ranks, threshold ties held by lower ranks) the tie quota and its start
// come from there instead of from this call's rows alone.
__global__ void __launch_bounds__(1024) scan_kernel(int B, int H, int nb, uint32_t kfree,
                                                    SelWs ws, int32_t* __restrict__ row_ptr,
                                                    const int64_t* __restrict__ offs) {
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  const int rows = H * nb;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int b = 0; b < B; ++b) {
    // the ties each row takes: the threshold's remaining count, by flat index
    uint32_t krem = 0;
    {
      // ties to take = kfree - (number of scores above the threshold in batch b)
      __shared__ int s_gt;
      if (threadIdx.x == 0) s_gt = 0;
      __syncthreads();
      int g = 0;
      for (int r = threadIdx.x; r < rows; r += 1024) g += ws.gt[(int64_t)b * rows + r];
      atomicAdd(&s_gt, g);
      __syncthreads();
      krem = kfree - (uint32_t)(offs ? offs[2 * b] : (int64_t)s_gt);
    }
    __shared__ int s_eqcarry;
    if (threadIdx.x == 0) {
      // ties held by lower ranks come first; more than the quota means none here
      const int64_t before = offs ? offs[2 * b + 1] : 0;
      s_eqcarry = before > (int64_t)krem ? (int)krem : (int)before;
    }
    __syncthreads();
    for (int r0 = 0; r0 < rows; r0 += 1024) {
      const int r = r0 + threadIdx.x;
      const int64_t row = (int64_t)b * rows + r;
      const int eq = r < rows ? ws.eq[row] : 0;
      const int gt = r < rows ? ws.gt[row] : 0;
      // exclusive scan of eq across the CTA
      int incl = eq;
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) s_warp[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        int v = s_warp[lane];
        for (int o = 1; o < 32; o <<= 1) {
          int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        s_warp[lane] = v;  // inclusive over warps
      }
      __syncthreads();
      const int before = s_eqcarry + (warp ? s_warp[warp - 1] : 0) + incl - eq;
      int take = (int)krem - before;
      take = take < 0 ? 0 : (take > eq ? eq : take);
      const int cnt = gt + take + 1;
      const int chunk_eq = s_warp[31];
      __syncthreads();
      // exclusive scan of cnt for row_ptr
      incl = r < rows ? cnt : 0;
      const int mine = incl;
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) s_warp[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        int v = s_warp[lane];
        for (int o = 1; o < 32; o <<= 1) {
          int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        s_warp[lane] = v;
      }
      __syncthreads();
      if (r < rows) {
        row_ptr[row] = s_carry + (warp ? s_warp[warp - 1] : 0) + incl - mine;
        ws.take[row] = take;
      }
      const int chunk_cnt = s_warp[31];
      __syncthreads();
      if (threadIdx.x == 0) {
        s_carry += chunk_cnt;
        s_eqcarry += chunk_eq;
      }
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) row_ptr[(int64_t)B * rows] = s_carry;
}

// grid: (row chunks, B); one warp per row writes its kept blocks in ascending j.
__global__ void __launch_bounds__(kThreads) write_kernel(const float* __restrict__ scores, int B,
                                                         int H, int nb, SelWs ws,
                                                         const int32_t* __restrict__ row_ptr,
                                                         int32_t* __restrict__ col_idx,
                                                         uint8_t* __restrict__ mask) {
  const int b = blockIdx.y;
  const uint32_t tau = ws.tau[b];
  const int lane = threadIdx.x % 32;
  const int rows = H * nb;
  for (int r = blockIdx.x * (kThreads / 32) + threadIdx.x / 32; r < rows;
       r += gridDim.x * (kThreads / 32)) {
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

// grid: B; per batch element this call's keys above the threshold and equal to
// it (totals[2b], totals[2b+1]).
__global__ void __launch_bounds__(kThreads) totals_kernel(int B, int H, int nb, SelWs ws,
                                                          int64_t* __restrict__ totals) {
  __shared__ unsigned long long s[2];
  const int b = blockIdx.x;
  if (threadIdx.x == 0) s[0] = s[1] = 0;
  __syncthreads();
  unsigned long long g = 0, e = 0;
  const int rows = H * nb;
  for (int r = threadIdx.x; r < rows; r += kThreads) {
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

size_t select_workspace_bytes(int B, int H, int nb) {
  const size_t R = (size_t)B * H * nb;
  return align256(sizeof(int) * (size_t)kPasses * B * kBins) + 3 * align256(sizeof(int) * R) +
         align256(sizeof(uint32_t) * (size_t)B);
}

cudaError_t launch_select(const float* scores, int B, int H, int nb, int64_t kb, int32_t* row_ptr,
                          int32_t* col_idx, uint8_t* mask, void* ws_raw, cudaStream_t st) {
  const int R = B * H * nb;
  SelWs ws = carve(ws_raw, B, R);
  const uint32_t kfree = (uint32_t)(kb - (int64_t)H * nb);
  const size_t nh = (size_t)kPasses * B * kBins;
  zero_kernel<<<(unsigned)((nh + 255) / 256), 256, 0, st>>>(ws.hist, nh);
  const int64_t per_b = (int64_t)H * nb * nb;
  int chunks = (int)((per_b / 4 + kThreads - 1) / kThreads);
  if (chunks < 1) chunks = 1;
  if (chunks > 148 * 4) chunks = 148 * 4;
  for (int p = 0; p < kPasses; ++p)
    hist_kernel<<<dim3(chunks, B), kThreads, 0, st>>>(scores, B, H, nb, kfree, p, ws);
  int rchunks = (H * nb + (kThreads / 32) - 1) / (kThreads / 32);
  if (rchunks > 148 * 8) rchunks = 148 * 8;
  count_kernel<<<dim3(rchunks, B), kThreads, 0, st>>>(scores, B, H, nb, kfree, ws);
  scan_kernel<<<1, 1024, 0, st>>>(B, H, nb, kfree, ws, row_ptr, nullptr);
  write_kernel<<<dim3(rchunks, B), kThreads, 0, st>>>(scores, B, H, nb, ws, row_ptr, col_idx,
                                                      mask);
  return cudaGetLastError();
}

// ------------------------------------------------- heads split over ranks
// The same selection in stages, for a sequence whose heads are split over
// ranks (contiguous head ranges in rank order, so flat order is rank order).
// Between the stages the caller sums the pass histograms over ranks and
// exchanges the per-rank totals; every stage re-derives the threshold from the
// summed histograms, so all ranks agree on it.

cudaError_t launch_select_shard_pass(const float* scores, int B, int H, int nb, int64_t kfree,
                                     int pass, void* ws_raw, cudaStream_t st) {
  const int R = B * H * nb;
  SelWs ws = carve(ws_raw, B, R);
  if (pass == 0) {
    const size_t nh = (size_t)kPasses * B * kBins;
    zero_kernel<<<(unsigned)((nh + 255) / 256), 256, 0, st>>>(ws.hist, nh);
  }
  const int64_t per_b = (int64_t)H * nb * nb;
  int chunks = (int)((per_b / 4 + kThreads - 1) / kThreads);
  if (chunks < 1) chunks = 1;
  if (chunks > 148 * 4) chunks = 148 * 4;
  hist_kernel<<<dim3(chunks, B), kThreads, 0, st>>>(scores, B, H, nb, (uint32_t)kfree, pass, ws);
  return cudaGetLastError();
}

cudaError_t launch_select_shard_count(const float* scores, int B, int H, int nb, int64_t kfree,
                                      void* ws_raw, int64_t* totals, cudaStream_t st) {
  const int R = B * H * nb;
  SelWs ws = carve(ws_raw, B, R);
  int rchunks = (H * nb + (kThreads / 32) - 1) / (kThreads / 32);
  if (rchunks > 148 * 8) rchunks = 148 * 8;
  count_kernel<<<dim3(rchunks, B), kThreads, 0, st>>>(scores, B, H, nb, (uint32_t)kfree, ws);
  totals_kernel<<<B, kThreads, 0, st>>>(B, H, nb, ws, totals);
  return cudaGetLastError();
}

cudaError_t launch_select_shard_finish(const float* scores, int B, int H, int nb, int64_t kfree,
                                       const int64_t* offs, void* ws_raw, int32_t* row_ptr,
                                       int32_t* col_idx, uint8_t* mask, cudaStream_t st) {
  const int R = B * H * nb;
  SelWs ws = carve(ws_raw, B, R);
  scan_kernel<<<1, 1024, 0, st>>>(B, H, nb, (uint32_t)kfree, ws, row_ptr, offs);
  int rchunks = (H * nb + (kThreads / 32) - 1) / (kThreads / 32);
  if (rchunks > 148 * 8) rchunks = 148 * 8;
  write_kernel<<<dim3(rchunks, B), kThreads, 0, st>>>(scores, B, H, nb, ws, row_ptr, col_idx,
                                                      mask);
  return cudaGetLastError();
}

size_t select_hist_offset(int B, int pass) { return sizeof(int) * (size_t)pass * B * kBins; }
size_t select_hist_count(int B) { return (size_t)B * kBins; }

}  // namespace sdl
