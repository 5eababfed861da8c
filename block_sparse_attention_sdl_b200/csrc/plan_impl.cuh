// Device code of the tile plan (pairing 64-token query blocks into 128-row
// tiles by kept-list overlap), shared by plan.cu and the fused anchor kernel
// of anchor.cu.  See plan.cu for the rule.
#pragma once
#include "internal.cuh"

namespace sdl {
namespace planimpl {
namespace {  // internal linkage in every translation unit that includes this


constexpr int kPlanThreads = 512;
constexpr int kPlanMaxNb = 256;

struct PlanSmem {
  static size_t bytes(int nb) {
    const int nw = (nb + 31) / 32;
    return sizeof(uint32_t) * (size_t)nb * nw      // kept-list bitmaps, word-major
           + sizeof(uint16_t) * (size_t)nb * nb    // pairwise intersections
           + sizeof(int) * 2 * (size_t)nb          // list lengths, visiting order
           + sizeof(int) * ((size_t)nb + 1)        // the head's row offsets
           + 16;
  }
};

// Block (head h, batch element b), any multiple of 32 threads; shared memory
// `psm` of PlanSmem::bytes(nb), 16-byte aligned.  NW >= ceil(nb / 32): the
// bitmap words (and lane chunks) the loops are unrolled for.
template <int NW>
__device__ __forceinline__ void plan_body_w(const int32_t* __restrict__ row_ptr,
                                            const int32_t* __restrict__ col_idx, int H, int nb,
                                            int n_qt, int32_t* __restrict__ plan, int h, int b,
                                            uint8_t* psm) {
  const int nthr = blockDim.x;
  const int nw = (nb + 31) / 32;
  uint32_t* bits = reinterpret_cast<uint32_t*>(psm);
  uint16_t* ov = reinterpret_cast<uint16_t*>(bits + (size_t)nb * nw);
  int* len = reinterpret_cast<int*>(ov + (size_t)nb * nb + ((nb * nb) & 1));
  int* order = len + nb;
  int* rp = order + nb;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int64_t r0 = ((int64_t)b * H + h) * nb;
  int32_t* out = plan + ((int64_t)b * H + h) * n_qt * 2;

  for (int x = tid; x < nb * nw; x += nthr) bits[x] = 0u;
  for (int x = tid; x <= nb; x += nthr) rp[x] = row_ptr[r0 + x];
  __syncthreads();
  // the head's entries as one flat range; an entry's row by binary search in rp
  {
    const int base = rp[0], n = rp[nb] - rp[0];
    for (int x = tid; x < n; x += nthr) {
      int lo = 0, hi = nb - 1;  // last row whose start is <= base + x
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rp[mid] <= base + x)
          lo = mid;
        else
          hi = mid - 1;
      }
      const int j = col_idx[base + x];
      if (j >= 0 && j < nb) atomicOr(&bits[(j / 32) * nb + lo], 1u << (j % 32));
    }
  }
  __syncthreads();
  for (int i = tid; i < nb; i += nthr) {
    int c = 0;
    for (int w = 0; w < nw; ++w) c += __popc(bits[w * nb + i]);
    len[i] = c;
  }
  __syncthreads();
  const int nwarps = nthr / 32;
  // intersections, one warp per row i: lanes read consecutive words of the
  // word-major bitmaps and write consecutive entries (no bank conflicts)
  for (int i = warp; i < nb; i += nwarps) {
    uint32_t bi[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) bi[w] = w < nw ? bits[w * nb + i] : 0u;
    for (int j = lane; j < nb; j += 32) {
      int c = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w)
        if (w < nw) c += __popc(bi[w] & bits[w * nb + j]);
      ov[i * nb + j] = (uint16_t)c;
    }
  }
  // visiting order: by descending list length, ties by lower index; the rank of
  // block i counts the blocks before it, 32 at a time by ballot
  for (int i = warp; i < nb; i += nwarps) {
    const int li = len[i];
    int rank = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const bool before = j < nb && (len[j] > li || (len[j] == li && j < i));
      rank += __popc(__ballot_sync(0xffffffffu, before));
    }
    if (lane == 0) order[rank] = i;
  }
  __syncthreads();
  if (warp == 0) {
    // lane owns the blocks j = lane + 32 c; bit c of `unpaired`: that block exists
    // and is not paired yet
    const int nc = (nb + 31) / 32;
    uint32_t unpaired = 0;
    for (int c = 0; c < nc; ++c)
      if (lane + 32 * c < nb) unpaired |= 1u << c;
    int p = 0;
    int i_next = order[0];
    for (int k = 0; k < nb; ++k) {
      const int i = i_next;
      if (k + 1 < nb) i_next = order[k + 1];
      // candidate keys of row i, (intersection + 1) << 16 | (0xFFFF - j): the
      // largest is the largest intersection, lowest index on ties.  They do not
      // depend on the pairing so far, so their loads leave the serial chain.
      uint32_t kj[NW];
#pragma unroll
      for (int c = 0; c < NW; ++c) {
        const int j = lane + 32 * c;
        kj[c] = (c < nc && j < nb)
                    ? ((uint32_t)ov[i * nb + j] + 1u) << 16 | (0xFFFFu - (uint32_t)j)
                    : 0u;
      }
      if (!((__shfl_sync(0xffffffffu, unpaired, i & 31) >> (i >> 5)) & 1u)) continue;
      if (lane == (i & 31)) unpaired &= ~(1u << (i >> 5));
      // the unpaired partner with the largest key; 0 when none is left
      uint32_t key = 0;
#pragma unroll
      for (int c = 0; c < NW; ++c)
        if ((unpaired >> c) & 1u) key = kj[c] > key ? kj[c] : key;
      key = __reduce_max_sync(0xffffffffu, key);
      const int best = key ? (int)(0xFFFFu - (key & 0xFFFFu)) : -1;
      if (best >= 0 && lane == (best & 31)) unpaired &= ~(1u << (best >> 5));
      if (lane == 0) {
        out[2 * p] = i;
        out[2 * p + 1] = best;
      }
      ++p;
    }
  }
  __syncthreads();  // shared memory may be reused by the block's next item
}

__device__ __forceinline__ void plan_body(const int32_t* __restrict__ row_ptr,
                                          const int32_t* __restrict__ col_idx, int H, int nb,
                                          int n_qt, int32_t* __restrict__ plan, int h, int b,
                                          uint8_t* psm) {
  static_assert(kPlanMaxNb == 256, "unrolled for at most 8 bitmap words");
  if (nb <= 32)
    plan_body_w<1>(row_ptr, col_idx, H, nb, n_qt, plan, h, b, psm);
  else if (nb <= 64)
    plan_body_w<2>(row_ptr, col_idx, H, nb, n_qt, plan, h, b, psm);
  else if (nb <= 128)
    plan_body_w<4>(row_ptr, col_idx, H, nb, n_qt, plan, h, b, psm);
  else
    plan_body_w<8>(row_ptr, col_idx, H, nb, n_qt, plan, h, b, psm);
}

}  // namespace
}  // namespace planimpl
}  // namespace sdl
