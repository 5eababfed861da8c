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
#include "plan_impl.cuh"
#include "select_impl.cuh"

namespace sdl {
namespace {

using namespace planimpl;

// grid (H, B); dynamic shared memory PlanSmem::bytes(nb); nb <= 32 * NW
template <int NW>
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ row_ptr,
                                                            const int32_t* __restrict__ col_idx,
                                                            int H, int nb, int n_qt,
                                                            int32_t* __restrict__ plan) {
  extern __shared__ __align__(16) uint8_t psm[];
  plan_body_w<NW>(row_ptr, col_idx, H, nb, n_qt, plan, blockIdx.x, blockIdx.y, psm);
}

template <int NW>
cudaError_t launch_plan_w(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int nb,
                          int32_t* plan, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];  // per device; the maximum is constant
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(plan_kernel<NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)PlanSmem::bytes(32 * NW));
  });
  if (e != cudaSuccess) return e;
  plan_kernel<NW><<<dim3(H, B), kPlanThreads, PlanSmem::bytes(nb), st>>>(row_ptr, col_idx, H, nb,
                                                                       (nb + 1) / 2, plan);
  return cudaGetLastError();
}

constexpr int kOrderThreads = 1024;
constexpr int kOrderBins = 2 * 1024 + 1;  // tile costs 0 .. 2 nb, nb <= 1024
// tiles whose costs are kept in shared memory between the two walks (16 bits
// each); beyond this the second walk recomputes them from the lists
constexpr int kOrderCached = 48 * 1024;
constexpr size_t kOrderCountBytes = 112 * 1024;  // per-warp bin counters, at most

// Warps that count their own chunk of the tiles: as many as the per-warp
// counters of nbins bins allow (at least one).
inline int order_warps(int nbins) {
  const int w = (int)(kOrderCountBytes / (sizeof(int) * (size_t)nbins));
  return w < 1 ? 1 : (w > kOrderThreads / 32 ? kOrderThreads / 32 : w);
}

// One CTA: the order in which the attention kernel takes its tiles, costliest
// first, so that the long tiles of heavy heads do not run last and leave the
// other SMs idle.  A tile's cost is the sum of its two query blocks' list
// lengths (an upper bound of the union it walks); a stable counting sort orders
// them (equal costs keep the tile order, so tiles of one head stay together and
// share its K and V in L2).  order[r] = the r-th tile to take.
//
// Warp w < W counts the costs of its contiguous chunk of tiles into its own
// row of counters; a scan over (cost descending, warp ascending) gives every
// (warp, cost) its first place; each warp then walks its chunk again in order,
// lanes of equal cost taking consecutive places in lane order.
__global__ void __launch_bounds__(kOrderThreads) order_kernel(const int32_t* __restrict__ row_ptr,
                                                              const int32_t* __restrict__ plan,
                                                              int BH, int nb, int n_qt, int W,
                                                              int32_t* __restrict__ order) {
  __shared__ int start[kOrderBins];
  __shared__ int s_warp[32];
  extern __shared__ __align__(16) int cnt_sm[];  // [W][nbins], then the costs (16 bits)
  const int n = BH * n_qt, tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int nbins = 2 * nb + 1;
  const bool cached = n <= kOrderCached;
  uint16_t* cost_sm = reinterpret_cast<uint16_t*>(cnt_sm + (size_t)W * nbins);
  auto cost_of = [&](int x) -> int {
    const int64_t r0 = (int64_t)(x / n_qt) * nb;
    int c = 0;
    for (int s = 0; s < 2; ++s) {
      const int qb = plan[2 * (int64_t)x + s];
      if (qb >= 0 && qb < nb) c += row_ptr[r0 + qb + 1] - row_ptr[r0 + qb];
    }
    return c < 0 ? 0 : (c >= nbins ? nbins - 1 : c);
  };
  const int chunk = (n + W - 1) / W;
  const int x0 = warp * chunk, x1 = x0 + chunk < n ? x0 + chunk : n;
  for (int c = tid; c < W * nbins; c += kOrderThreads) cnt_sm[c] = 0;
  __syncthreads();
  if (warp < W)
    for (int x = x0 + lane; x < x1; x += 32) {
      const int c = cost_of(x);
      if (cached) cost_sm[x] = (uint16_t)c;
      atomicAdd(&cnt_sm[warp * nbins + c], 1);
    }
  __syncthreads();
  // per cost: the warps' counts into exclusive offsets, the total into start[]
  for (int c = tid; c < nbins; c += kOrderThreads) {
    int s = 0;
    for (int w = 0; w < W; ++w) {
      const int v = cnt_sm[w * nbins + c];
      cnt_sm[w * nbins + c] = s;
      s += v;
    }
    start[c] = s;
  }
  __syncthreads();
  // first place of each cost, costs in descending order: thread t owns bins
  // nbins - 1 - 3t, -3t-1, -3t-2
  int cnt[3], local = 0;
  for (int y = 0; y < 3; ++y) {
    const int c = nbins - 1 - 3 * tid - y;
    cnt[y] = c >= 0 ? start[c] : 0;
    local += cnt[y];
  }
  int total = 0;
  int pos = selimpl::block_excl_scan(local, s_warp, total);
  for (int y = 0; y < 3; ++y) {
    const int c = nbins - 1 - 3 * tid - y;
    if (c >= 0) start[c] = pos;
    pos += cnt[y];
  }
  __syncthreads();
  if (warp < W) {
    int* run = cnt_sm + warp * nbins;  // this warp's next place per cost, less start[]
    for (int base = x0; base < x1; base += 32) {
      const int x = base + lane;
      const int c = x < x1 ? (cached ? (int)cost_sm[x] : cost_of(x)) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      if (x < x1) order[start[c] + run[c] + rank] = x;
      __syncwarp();
      if (x < x1 && lane == __ffs(peers) - 1) run[c] += __popc(peers);
      __syncwarp();
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
  if (nb <= 32) return launch_plan_w<1>(row_ptr, col_idx, B, H, nb, plan, st);
  if (nb <= 64) return launch_plan_w<2>(row_ptr, col_idx, B, H, nb, plan, st);
  if (nb <= 128) return launch_plan_w<4>(row_ptr, col_idx, B, H, nb, plan, st);
  return launch_plan_w<8>(row_ptr, col_idx, B, H, nb, plan, st);
}

cudaError_t launch_tile_order(const int32_t* row_ptr, const int32_t* plan, int B, int H, int nb,
                              int32_t* order, cudaStream_t st) {
  if (nb < 1 || nb > (kOrderBins - 1) / 2) return cudaErrorInvalidValue;
  const int n = B * H * ((nb + 1) / 2);
  const int nbins = 2 * nb + 1, W = order_warps(nbins);
  const size_t smem = sizeof(int) * (size_t)W * nbins +
                      (n <= kOrderCached ? sizeof(uint16_t) * (size_t)n : 0);
  static std::atomic<bool> attr_set[64];  // per device
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(kOrderCountBytes + sizeof(uint16_t) * kOrderCached));
  });
  if (e != cudaSuccess) return e;
  order_kernel<<<1, kOrderThreads, smem, st>>>(row_ptr, plan, B * H, nb, (nb + 1) / 2, W,
                                               order);
  return cudaGetLastError();
}

}  // namespace sdl
