// Tile plan for 64-token blocks: which two query blocks share a 128-row
// tensor-core tile of the attention kernel.
//
// The attention kernel's tile covers two query blocks and walks the union of
// their kept lists, so its work is the union's size, not the sum of the two
// lists.  Per (b, h) this kernel pairs the query blocks greedily by overlap:
// blocks in order of descending list length (ties: lower index first), each
// still unpaired block taking the unpaired block with the largest
// intersection of kept lists (ties: lower index).  Output: int32
// [B, H, ceil(nb/2), 2], tile p of (b, h) = query blocks (plan[2p],
// plan[2p+1]); the second entry is -1 for the single block left when nb is
// odd.  Heads with more than kPlanMaxNb blocks get adjacent pairs (2p, 2p+1).
// The plan is a schedule only: attention results do not depend on it beyond
// fp32 summation order.
#include "internal.cuh"

namespace sdl {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanMaxNb = 256;

struct PlanSmem {
  static size_t bytes(int nb) {
    const int nw = (nb + 31) / 32;
    return sizeof(uint32_t) * (size_t)nb * nw      // kept-list bitmaps
           + sizeof(uint16_t) * (size_t)nb * nb    // pairwise intersections
           + sizeof(int) * 2 * (size_t)nb          // list lengths, visiting order
           + (size_t)nb + 16;                      // paired flags
  }
};

// grid (H, B); dynamic shared memory PlanSmem::bytes(nb)
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ row_ptr,
                                                            const int32_t* __restrict__ col_idx,
                                                            int H, int nb, int n_qt,
                                                            int32_t* __restrict__ plan) {
  extern __shared__ __align__(16) uint8_t psm[];
  const int nw = (nb + 31) / 32;
  uint32_t* bits = reinterpret_cast<uint32_t*>(psm);
  uint16_t* ov = reinterpret_cast<uint16_t*>(bits + (size_t)nb * nw);
  int* len = reinterpret_cast<int*>(ov + (size_t)nb * nb + ((nb * nb) & 1));
  int* order = len + nb;
  volatile uint8_t* used = reinterpret_cast<uint8_t*>(order + nb);
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int64_t r0 = ((int64_t)b * H + h) * nb;
  int32_t* out = plan + ((int64_t)b * H + h) * n_qt * 2;

  for (int x = tid; x < nb * nw; x += kPlanThreads) bits[x] = 0u;
  for (int x = tid; x < nb; x += kPlanThreads) used[x] = 0;
  __syncthreads();
  for (int i = warp; i < nb; i += kPlanThreads / 32) {
    const int beg = row_ptr[r0 + i], end = row_ptr[r0 + i + 1];
    for (int x = beg + lane; x < end; x += 32) {
      const int j = col_idx[x];
      if (j >= 0 && j < nb) atomicOr(&bits[i * nw + j / 32], 1u << (j % 32));
    }
  }
  __syncthreads();
  for (int i = tid; i < nb; i += kPlanThreads) {
    int c = 0;
    for (int w = 0; w < nw; ++w) c += __popc(bits[i * nw + w]);
    len[i] = c;
  }
  for (int x = tid; x < nb * nb; x += kPlanThreads) {
    const int i = x / nb, j = x % nb;
    int c = 0;
    for (int w = 0; w < nw; ++w) c += __popc(bits[i * nw + w] & bits[j * nw + w]);
    ov[x] = (uint16_t)c;
  }
  __syncthreads();
  for (int i = tid; i < nb; i += kPlanThreads) {
    int rank = 0;
    for (int j = 0; j < nb; ++j) rank += (len[j] > len[i]) || (len[j] == len[i] && j < i);
    order[rank] = i;
  }
  __syncthreads();
  if (warp == 0) {
    int p = 0;
    for (int k = 0; k < nb; ++k) {
      const int i = order[k];
      if (used[i]) continue;
      __syncwarp();
      if (lane == 0) used[i] = 1;
      __syncwarp();
      // unpaired partner of largest intersection, lowest index on ties
      int best = -1, bv = -1;
      for (int j = lane; j < nb; j += 32) {
        if (used[j]) continue;
        const int v = ov[i * nb + j];
        if (v > bv) {
          bv = v;
          best = j;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const int v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const int b2 = __shfl_xor_sync(0xffffffffu, best, o);
        if (v2 > bv || (v2 == bv && b2 >= 0 && (best < 0 || b2 < best))) {
          bv = v2;
          best = b2;
        }
      }
      if (lane == 0) {
        if (best >= 0) used[best] = 1;
        out[2 * p] = i;
        out[2 * p + 1] = best;
      }
      __syncwarp();
      ++p;
    }
  }
}

// Adjacent pairs (2p, 2p+1), for heads too long for the greedy plan.
__global__ void adjacent_plan_kernel(int64_t n_tiles, int nb, int n_qt, int32_t* plan) {
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n_tiles;
       x += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(x % n_qt);
    plan[2 * x] = 2 * p;
    plan[2 * x + 1] = 2 * p + 1 < nb ? 2 * p + 1 : -1;
  }
}

}  // namespace

cudaError_t launch_plan(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int nb,
                        int32_t* plan, cudaStream_t st) {
  const int n_qt = (nb + 1) / 2;
  if (nb > kPlanMaxNb) {
    const int64_t n_tiles = (int64_t)B * H * n_qt;
    const int grid = (int)((n_tiles + 255) / 256 < 1184 ? (n_tiles + 255) / 256 : 1184);
    adjacent_plan_kernel<<<grid, 256, 0, st>>>(n_tiles, nb, n_qt, plan);
    return cudaGetLastError();
  }
  const size_t smem = PlanSmem::bytes(nb);
  static bool attr_set = false;  // the attribute is per function; the maximum is constant
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PlanSmem::bytes(kPlanMaxNb));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  plan_kernel<<<dim3(H, B), kPlanThreads, smem, st>>>(row_ptr, col_idx, H, nb, n_qt, plan);
  return cudaGetLastError();
}

}  // namespace sdl
