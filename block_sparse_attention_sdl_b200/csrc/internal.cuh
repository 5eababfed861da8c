// Declarations shared by the translation units of libsdl.
#pragma once
#include <atomic>

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sdl.h"

namespace sdl {

// Device status word bits (set by kernels, read by sdl_last_device_status).
// kDevOverlap: two attention launches in flight shared one tile counter.
enum : int { kDevTimeout = 1, kDevBadMask = 2, kDevOverlap = 4 };

// Sites of bad-mask reports.  The word after the status word records the first
// report since the last read: site << 24 | the low 24 bits of the offending value.
enum : int {
  kBadPlanEntry = 1,    // a tile plan entry outside [-1, nb)
  kBadListEntry = 2,    // a CSR entry out of range or not ascending (value: the entry)
  kBadRecord = 3,       // a tile-lists record's tile or length (value: the tile)
  kBadRecordRows = 4,   // a tile-lists record's first tokens (value: t0)
  kBadRecordEntry = 5,  // a tile-lists entry's key sub-block (value: the entry)
  kBadOrderEntry = 6,   // a take-order entry, attention kernel (value: the entry)
  kBadListsOrder = 7,   // a take-order entry, tile-lists kernel (value: the entry)
  kBadSimtEntry = 8,    // a CSR entry, fp32 kernel (value: the entry)
};

__device__ __forceinline__ void report_bad_mask(int* status, int site, int value) {
  atomicOr(status, kDevBadMask);
  atomicCAS(status + 1, 0, (site << 24) | (value & 0xFFFFFF));
}

// Wall-time bound for every spin wait inside a kernel.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

int* device_status_ptr();  // the library's device status word and its detail word

// List entries handed to the attention kernels: 64-token key sub-block index
// in the low 16 bits, and in bits 16..17 which halves (query rows 0..63,
// 64..127) of a 128-row query tile keep it.
constexpr int kSubBlock = 64;

// Runs `set` (setting a kernel's attributes) once per device for the static
// flags `done` of one call site; a failure is returned and retried next time.
template <typename F>
inline cudaError_t once_per_device(std::atomic<bool> (&done)[64], F&& set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev].load()) return cudaSuccess;
  e = set();
  if (e == cudaSuccess) done[dev].store(true);
  return e;
}

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const int32_t* row_ptr;  // null: dense
  const int32_t* col_idx;
  const int32_t* plan;     // tile plan for 64-token blocks (null: adjacent pairs)
  const int32_t* order;    // order of taking the plan's tiles (null: plan order)
  const int32_t* lists;    // prebuilt tile lists in take order (null: built in the kernel)
  int B, H, Hkv, L, d, block, nb;
  int Lk;  // key (and value) tokens: L, or the gathered columns of column-sparse attention
  int64_t qs[3], ks[3], vs[3], os[3];
  float scale_log2;  // scale * log2(e)
  float scale;
  int* status;
};

cudaError_t launch_pool(const void* q, const void* k, const sdl_shape& s, float* qbar, float* kbar,
                        cudaStream_t st);
cudaError_t launch_scores(const float* qbar, const float* kbar, const sdl_shape& s, float scale,
                          float* scores, cudaStream_t st);
cudaError_t launch_select(const float* scores, int B, int H, int nb, int64_t kb, int32_t* row_ptr,
                          int32_t* col_idx, uint8_t* mask, void* ws, cudaStream_t st);
size_t select_workspace_bytes(int B, int H, int nb);
// staged selection for heads split over ranks (select.cu)
cudaError_t launch_select_shard_pass(const float* scores, int B, int H, int nb, int64_t kfree,
                                     int pass, void* ws, cudaStream_t st);
cudaError_t launch_select_shard_count(const float* scores, int B, int H, int nb, int64_t kfree,
                                      void* ws, int64_t* totals, cudaStream_t st);
cudaError_t launch_select_shard_finish(const float* scores, int B, int H, int nb, int64_t kfree,
                                       const int64_t* offs, void* ws, int32_t* row_ptr,
                                       int32_t* col_idx, uint8_t* mask, cudaStream_t st);
// fused anchor step (anchor.cu): scores, selection and (plan != nullptr) the
// tile plan in one cooperative launch; `bar` holds anchor_barrier_bytes()
cudaError_t launch_anchor(const void* q, const void* k, const sdl_shape& s, float scale,
                          int64_t kb, float* qbar, float* kbar, float* scores, void* sel_ws,
                          int32_t* row_ptr, int32_t* col_idx, int32_t* plan, unsigned* bar,
                          int* status, cudaStream_t st);
size_t anchor_barrier_bytes();
// column-sparse attention (col.cu)
size_t col_partial_bytes(const sdl_shape& s);
cudaError_t launch_col_scores(const void* k, const sdl_shape& s, float scale, const float* qbar,
                              float2* part, float2* stats, float* S, cudaStream_t st);
cudaError_t launch_col_select(const float* S, int BH, int L, int Lc, int32_t* cols,
                              cudaStream_t st);
cudaError_t launch_col_gather(const void* k, const void* v, const sdl_shape& s,
                              const int32_t* cols, int Lc, void* kc, void* vc, cudaStream_t st);
size_t tile_lists_bytes(int64_t n_items, int Lk);
cudaError_t launch_tile_lists(const AttnArgs& a, int32_t* lists, cudaStream_t st);
cudaError_t launch_tile_order(const int32_t* row_ptr, const int32_t* plan, int B, int H, int nb,
                              int32_t* order, cudaStream_t st);
// self-check of the bounded waits (selfcheck.cu)
cudaError_t launch_wait_check(uint64_t limit_ns, int* status, cudaStream_t st);
size_t select_hist_offset(int B, int pass);
size_t select_hist_count(int B);
cudaError_t launch_attn_tc(const AttnArgs& a, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, const CUtensorMap* to, cudaStream_t st);
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_plan(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int nb,
                        int32_t* plan, cudaStream_t st);

}  // namespace sdl
