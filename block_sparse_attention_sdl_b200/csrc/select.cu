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
#include "select_impl.cuh"

namespace sdl {
namespace {

using namespace selimpl;

__global__ void zero_kernel(int* p, size_t n) {
  for (size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x; x < n;
       x += (size_t)gridDim.x * blockDim.x)
    p[x] = 0;
}

// grid: (chunks, B)
__global__ void __launch_bounds__(kThreads) hist_kernel(const float* __restrict__ scores, int B,
                                                        int H, int nb, uint32_t kfree, int pass,
                                                        SelWs ws) {
  hist_body(scores, B, H, nb, kfree, pass, ws, blockIdx.x, gridDim.x, blockIdx.y);
}

// grid: (row chunks, B)
__global__ void __launch_bounds__(kThreads) count_kernel(const float* __restrict__ scores, int B,
                                                         int H, int nb, uint32_t kfree,
                                                         SelWs ws) {
  count_body(scores, B, H, nb, kfree, ws, blockIdx.x, gridDim.x, blockIdx.y);
}

// one CTA of 1024 threads
__global__ void __launch_bounds__(1024) scan_kernel(int B, int H, int nb, uint32_t kfree,
                                                    SelWs ws, int32_t* __restrict__ row_ptr,
                                                    const int64_t* __restrict__ offs) {
  scan_body(B, H, nb, kfree, ws, row_ptr, offs);
}

// grid: (row chunks, B)
__global__ void __launch_bounds__(kThreads) write_kernel(const float* __restrict__ scores, int B,
                                                         int H, int nb, SelWs ws,
                                                         const int32_t* __restrict__ row_ptr,
                                                         int32_t* __restrict__ col_idx,
                                                         uint8_t* __restrict__ mask) {
  write_body(scores, B, H, nb, ws, row_ptr, col_idx, mask, blockIdx.x, gridDim.x, blockIdx.y);
}

// grid: B
__global__ void __launch_bounds__(kThreads) totals_kernel(int B, int H, int nb, SelWs ws,
                                                          int64_t* __restrict__ totals) {
  totals_body(B, H, nb, ws, totals, blockIdx.x);
}

}  // namespace

size_t select_workspace_bytes(int B, int H, int nb) {
  return selimpl::carve_bytes(B, (size_t)B * H * nb);
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
