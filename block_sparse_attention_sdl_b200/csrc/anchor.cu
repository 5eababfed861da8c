// The anchor step of the Step-dLLM abstract in one launch: block scores,
// mask selection under the head-adaptive global budget, and the tile plan of
// the attention kernel.
//
// The separate kernels of scores.cu, select.cu and plan.cu take one launch per
// phase (ten at an anchor); at the 2K and 8K workloads most of their time is
// launch and ramp latency, not work.  Here one persistent cooperative grid (all
// blocks resident) runs the phases back to back, separated by grid barriers:
//   pooling -> | scores, each block histogramming the first digit of the rows
//   it wrote -> | digit pass 1 -> | pass 2 -> | per-row counts over contiguous
//   row chunks -> | each chunk: offsets from the earlier chunks' totals, tie
//   quotas, list compaction -> | tile plan
// Results are bit for bit those of the separate calls (the same scoring
// bodies and order of every floating-point operation; the same keys and tie
// rule in the selection).  Every barrier wait is bounded: on timeout the grid
// raises the device status word and every block returns.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "plan_impl.cuh"
#include "ptx.cuh"
#include "scores_impl.cuh"
#include "select_impl.cuh"

namespace sdl {
namespace {

using planimpl::kPlanMaxNb;
using planimpl::plan_body;
using planimpl::PlanSmem;
using scimpl::kTI;
using scimpl::PoolTensor;
using scimpl::pool_body;
using scimpl::score_body;
using scimpl::score_rows_offset;
using scimpl::score_smem_bytes;
using selimpl::count_chunk_body;
using selimpl::finish_chunk_body;
using selimpl::hist0_rows_body;
using selimpl::hist_body;
using selimpl::kBins;
using selimpl::kPasses;
using selimpl::SelWs;

constexpr int kAnchorThreads = 256;  // the selection bodies need exactly 256
// the first digit's bins sit in the score staging, in front of the kept rows
static_assert(scimpl::kTI * (64 + 4) * sizeof(float) + scimpl::kTJ * (64 + 4) * sizeof(float) >=
                  sizeof(int) * selimpl::kBins,
              "bins overlap the kept score rows");
constexpr int kBarriers = 8;

struct AnchorArgs {
  PoolTensor tq, tk;
  int B, H, Hkv, L, d, bs, nb, n_qt;
  float* qbar;
  float* kbar;
  float* scores;
  float scale;
  uint32_t kfree;
  SelWs ws;
  int32_t* row_ptr;
  int32_t* col_idx;
  int32_t* plan;    // nullable
  unsigned* bar;    // kBarriers arrival counters, zero at launch
  int* status;
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid barrier k: every block arrives once, then waits until all have, for at
// most the wait limit (or until another block gave up).  False: give up.
__device__ bool grid_barrier(const AnchorArgs& a, int k, volatile int* give_up) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(&a.bar[k], 1u);
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(&a.bar[k]) < gridDim.x) {
      if ((*(volatile int*)a.status & kDevTimeout) || globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(a.status, kDevTimeout);
        *give_up = 1;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
  return *give_up == 0;
}

template <typename T>
__global__ void __launch_bounds__(kAnchorThreads, 1) anchor_kernel(AnchorArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ volatile int give_up;
  if (threadIdx.x == 0) give_up = 0;
  const int tid = threadIdx.x, nblk = gridDim.x;
  // the radix histograms start from zero (first read after the second barrier)
  const size_t nh = (size_t)kPasses * a.B * kBins;
  for (size_t x = (size_t)blockIdx.x * kAnchorThreads + tid; x < nh;
       x += (size_t)nblk * kAnchorThreads)
    a.ws.hist[x] = 0;

  // ---- block means of Q and K
  pool_body<T, 16, true>(a.tq, a.tk, a.B, a.L, a.d, a.bs, blockIdx.x, nblk);
  if (!grid_barrier(a, 0, &give_up)) return;

  // ---- pooled products and row softmax: items (query-block tile, head, batch);
  // each block then adds its rows to the first digit's histogram
  const int ntile = (a.nb + kTI - 1) / kTI;
  for (int v = blockIdx.x; v < ntile * a.H * a.B; v += nblk) {
    const int ti = v % ntile, h = (v / ntile) % a.H, b = v / (ntile * a.H);
    float* sm = reinterpret_cast<float*>(dsm);
    score_body<true>(a.qbar, a.kbar, a.scores, a.H, a.Hkv, a.nb, a.d, a.scale, ti, h, b, sm);
    // the item's rows stay in shared memory; the bins take the staging in front
    const int i0 = ti * kTI, nrows = a.nb - i0 < kTI ? a.nb - i0 : kTI;
    hist0_rows_body(sm + score_rows_offset(a.d), nrows, a.nb, i0, a.kfree, a.ws, b,
                    reinterpret_cast<int*>(dsm));
  }
  if (!grid_barrier(a, 1, &give_up)) return;

  // ---- radix select: the other two digit passes over every sequence's scores
  const int nck = nblk / a.B > 0 ? nblk / a.B : 1;  // chunks per sequence
  for (int p = 1; p < kPasses; ++p) {
    for (int v = blockIdx.x; v < nck * a.B; v += nblk)
      hist_body(a.scores, a.B, a.H, a.nb, a.kfree, p, a.ws, v % nck, nck, v / nck);
    if (!grid_barrier(a, 1 + p, &give_up)) return;
  }
  // ---- per-row counts over contiguous row chunks, then every chunk's offsets
  // from the earlier chunks' totals, tie quotas and lists
  const int rows = a.H * a.nb;
  const int ncx = nck < rows ? nck : rows;
  for (int v = blockIdx.x; v < ncx * a.B; v += nblk)
    count_chunk_body(a.scores, a.B, a.H, a.nb, a.kfree, a.ws, v % ncx, ncx, v / ncx);
  if (!grid_barrier(a, 4, &give_up)) return;
  for (int v = blockIdx.x; v < ncx * a.B; v += nblk)
    finish_chunk_body(a.scores, a.B, a.H, a.nb, a.ws, a.row_ptr, a.col_idx, v % ncx, ncx,
                      v / ncx);
  if (a.plan == nullptr) return;

  // ---- tile plan (needs every list of a head)
  if (!grid_barrier(a, 5, &give_up)) return;
  if (a.nb <= kPlanMaxNb) {
    for (int v = blockIdx.x; v < a.H * a.B; v += nblk)
      plan_body(a.row_ptr, a.col_idx, a.H, a.nb, a.n_qt, a.plan, v % a.H, v / a.H, dsm);
  } else {
    // heads too long for the greedy plan: adjacent pairs (2p, 2p+1)
    const int64_t n_tiles = (int64_t)a.B * a.H * a.n_qt;
    for (int64_t x = (int64_t)blockIdx.x * kAnchorThreads + tid; x < n_tiles;
         x += (int64_t)nblk * kAnchorThreads) {
      const int p = (int)(x % a.n_qt);
      a.plan[2 * x] = 2 * p;
      a.plan[2 * x + 1] = 2 * p + 1 < a.nb ? 2 * p + 1 : -1;
    }
  }
}

template <typename T>
cudaError_t launch_anchor_t(AnchorArgs& a, size_t smem, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // per device: the shared-memory size last configured and the grid it gives
  // ((smem << 24) | grid; 0: none yet), so that steady calls make no queries
  static std::atomic<uint64_t> config[64];
  const uint64_t c = config[dev].load();
  int grid = (int)(c & 0xFFFFFFu);
  if (c == 0 || (c >> 24) != (uint64_t)smem) {
    e = cudaFuncSetAttribute(anchor_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, anchor_kernel<T>, kAnchorThreads,
                                                      smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // every block resident (the barriers need it); two per SM keep HBM busy
    // while pooling
    grid = sms * (per_sm < 2 ? per_sm : 2);
    config[dev].store(((uint64_t)smem << 24) | (uint64_t)grid);
  }
  e = cudaMemsetAsync(a.bar, 0, sizeof(unsigned) * kBarriers, st);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel((const void*)anchor_kernel<T>, dim3(grid),
                                     dim3(kAnchorThreads), args, smem, st);
}

}  // namespace

size_t anchor_barrier_bytes() { return 256; }

cudaError_t launch_anchor(const void* q, const void* k, const sdl_shape& s, float scale,
                          int64_t kb, float* qbar, float* kbar, float* scores, void* sel_ws,
                          int32_t* row_ptr, int32_t* col_idx, int32_t* plan, unsigned* bar,
                          int* status, cudaStream_t st) {
  const int nb = s.L / s.block;
  const int V = s.dtype == SDL_BF16 ? 8 : 4;
  const int per_warp = 32 * V;
  AnchorArgs a;
  a.tq = PoolTensor{q, qbar, s.H, (s.H * s.d + per_warp - 1) / per_warp, s.q_strides[0],
                    s.q_strides[1], s.q_strides[2]};
  a.tk = PoolTensor{k, kbar, s.H_kv, (s.H_kv * s.d + per_warp - 1) / per_warp, s.k_strides[0],
                    s.k_strides[1], s.k_strides[2]};
  a.B = s.B;
  a.H = s.H;
  a.Hkv = s.H_kv;
  a.L = s.L;
  a.d = s.d;
  a.bs = s.block;
  a.nb = nb;
  a.n_qt = (nb + 1) / 2;
  a.qbar = qbar;
  a.kbar = kbar;
  a.scores = scores;
  a.scale = scale;
  a.kfree = (uint32_t)(kb - (int64_t)s.H * nb);
  a.ws = selimpl::carve(sel_ws, s.B, s.B * s.H * nb);
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.plan = plan;
  a.bar = bar;
  a.status = status;
  size_t smem = score_smem_bytes(nb, s.d);
  if (plan && nb <= kPlanMaxNb && PlanSmem::bytes(nb) > smem) smem = PlanSmem::bytes(nb);
  if (s.dtype == SDL_BF16) return launch_anchor_t<__nv_bfloat16>(a, smem, st);
  return launch_anchor_t<float>(a, smem, st);
}

}  // namespace sdl
