// extern "C" entry points of libsdl: argument validation, budget arithmetic,
// TMA descriptor encoding, launches and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "internal.cuh"

namespace sdl {

// [0]: status bits; [1]: the first bad-mask report's site and value
__device__ int g_device_status[2];

namespace {

thread_local int t_last_cuda_error = 0;
thread_local int t_last_device_detail = 0;

sdl_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = (int)e;
  return SDL_ERR_CUDA;
}

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every call.  Returns SDL_OK or the error to report.
sdl_status check_shape(const sdl_shape* s) {
  if (!s) return SDL_ERR_INVALID_ARG;
  if (s->B <= 0 || s->H <= 0 || s->H_kv <= 0 || s->L <= 0 || s->d <= 0 || s->block <= 0)
    return SDL_ERR_INVALID_ARG;
  if (s->H % s->H_kv) return SDL_ERR_INVALID_ARG;
  if (s->dtype != SDL_BF16 && s->dtype != SDL_FP32) return SDL_ERR_INVALID_ARG;
  if (s->block != 64 && s->block != 128) return SDL_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return SDL_ERR_UNSUPPORTED;
  if (s->L % s->block) return SDL_ERR_UNSUPPORTED;
  if (s->L > 65536) return SDL_ERR_UNSUPPORTED;
  if ((int64_t)s->B * s->H * (s->L / s->block) * (s->L / s->block) >= (int64_t)1 << 31)
    return SDL_ERR_UNSUPPORTED;
  return SDL_OK;
}

// Strides (b, t, h) in elements of a [B, T, heads, d] tensor: non-negative
// multiples of 16 bytes, and nonzero on every axis with more than one index.
// A zero stride there (a broadcast view, e.g. expand along heads) would make
// distinct rows alias one address, which the TMA tensor maps cannot express.
sdl_status check_strides(const int64_t* st, int dtype, int B, int T, int heads) {
  const int64_t q = dtype == SDL_BF16 ? 8 : 4;  // elements per 16 bytes
  const int size[3] = {B, T, heads};
  for (int i = 0; i < 3; ++i) {
    if (st[i] < 0 || st[i] % q) return SDL_ERR_INVALID_ARG;
    if (st[i] == 0 && size[i] > 1) return SDL_ERR_INVALID_ARG;
  }
  return SDL_OK;
}

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / sqrtf((float)d); }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D map over a [B, L, heads, d] bf16 tensor: dims (d, t, h, b), box of
// `box_d` d-columns x `box_t` tokens, zero fill out of range.  Loads use
// 64 x 64 boxes with 128-byte swizzle, the output stores 32 x 32 with 64-byte
// swizzle.
bool encode_bf16_map(CUtensorMap* map, const void* base, const sdl_shape& s, int heads,
                     const int64_t* st, cuuint32_t box_d = 64, cuuint32_t box_t = 64,
                     CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B, int tokens = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)(tokens > 0 ? tokens : s.L),
                        (cuuint64_t)heads, (cuuint64_t)s.B};
  cuuint64_t strides[3] = {(cuuint64_t)st[1] * 2, (cuuint64_t)st[2] * 2, (cuuint64_t)st[0] * 2};
  // check_strides admits a zero stride only on an axis of one index, whose
  // coordinate is always 0; the map still wants a nonzero multiple of 16 there
  for (int i = 0; i < 3; ++i)
    if (strides[i] == 0) strides[i] = 16;
  cuuint32_t box[4] = {box_d, box_t, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Lk: key and value tokens (0: L, the same as the queries).
sdl_status attn_common(const void* q, const void* k, const void* v, const sdl_shape* shape,
                       const int32_t* row_ptr, const int32_t* col_idx, const int32_t* plan,
                       float scale, void* o, float* lse, void* stream, int Lk = 0,
                       const int32_t* order = nullptr, const int32_t* lists = nullptr) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (!q || !k || !v || !o) return SDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return SDL_ERR_INVALID_ARG;
  const int lk = Lk > 0 ? Lk : s.L;
  if ((e = check_strides(s.q_strides, s.dtype, s.B, s.L, s.H)) ||
      (e = check_strides(s.k_strides, s.dtype, s.B, lk, s.H_kv)) ||
      (e = check_strides(s.v_strides, s.dtype, s.B, lk, s.H_kv)) ||
      (e = check_strides(s.o_strides, s.dtype, s.B, s.L, s.H)))
    return e;
  int* status = device_status_ptr();
  if (!status) return SDL_ERR_CUDA;
  AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.plan = (row_ptr && s.block == 64) ? plan : nullptr;
  a.order = a.plan ? order : nullptr;
  a.lists = lists;
  a.B = s.B;
  a.H = s.H;
  a.Hkv = s.H_kv;
  a.L = s.L;
  a.d = s.d;
  a.block = s.block;
  a.nb = s.L / s.block;
  a.Lk = Lk > 0 ? Lk : s.L;
  for (int i = 0; i < 3; ++i) {
    a.qs[i] = s.q_strides[i];
    a.ks[i] = s.k_strides[i];
    a.vs[i] = s.v_strides[i];
    a.os[i] = s.o_strides[i];
  }
  a.scale = resolve_scale(scale, s.d);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.status = status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t ce;
  if (s.dtype == SDL_BF16) {
    CUtensorMap tq, tk, tv, to;
    if (!encode_bf16_map(&tq, q, s, s.H, s.q_strides) ||
        !encode_bf16_map(&tk, k, s, s.H_kv, s.k_strides, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                         a.Lk) ||
        !encode_bf16_map(&tv, v, s, s.H_kv, s.v_strides, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                         a.Lk) ||
        !encode_bf16_map(&to, o, s, s.H, s.o_strides, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return cuda_fail(cudaErrorInvalidValue);
    ce = launch_attn_tc(a, &tq, &tk, &tv, &to, st);
  } else {
    ce = launch_attn_simt(a, st);
  }
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

}  // namespace

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

}  // namespace sdl

using namespace sdl;

// Arguments of the tile-list kernel for a 64-token-block mask.
static AttnArgs lists_args(const sdl_shape& s, const int32_t* row_ptr, const int32_t* col_idx,
                    const int32_t* plan, const int32_t* order, int* status) {
  AttnArgs a{};
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.plan = plan;
  a.order = order;
  a.lists = nullptr;
  a.B = s.B;
  a.H = s.H;
  a.Hkv = s.H_kv;
  a.L = s.L;
  a.d = s.d;
  a.block = s.block;
  a.nb = s.L / s.block;
  a.Lk = s.L;
  a.status = status;
  return a;
}

extern "C" {

int64_t sdl_mask_budget(const sdl_shape* shape, double sparsity) {
  if (check_shape(shape) != SDL_OK) return -1;
  if (!(sparsity >= 0.0 && sparsity < 1.0)) return -1;
  const int64_t nb = shape->L / shape->block;
  const double per = (double)shape->H * (double)nb * (double)nb;
  const int64_t kb = (int64_t)floor((1.0 - sparsity) * per + 0.5);
  if (kb < (int64_t)shape->H * nb) return -1;
  return kb * shape->B;
}

size_t sdl_scores_workspace_bytes(const sdl_shape* shape) {
  if (check_shape(shape) != SDL_OK) return 0;
  const size_t nb = shape->L / shape->block;
  return align256(sizeof(float) * shape->B * shape->H * nb * shape->d) +
         align256(sizeof(float) * shape->B * shape->H_kv * nb * shape->d);
}

size_t sdl_select_workspace_bytes(const sdl_shape* shape) {
  if (check_shape(shape) != SDL_OK) return 0;
  return select_workspace_bytes(shape->B, shape->H, shape->L / shape->block);
}

size_t sdl_select_workspace_bytes_scoped(const sdl_shape* shape, int scope) {
  if (scope == SDL_BUDGET_SEQUENCE) return sdl_select_workspace_bytes(shape);
  if (scope != SDL_BUDGET_HEAD || check_shape(shape) != SDL_OK) return 0;
  // every head is its own single-head sequence
  return select_workspace_bytes(shape->B * shape->H, 1, shape->L / shape->block);
}

int64_t sdl_mask_budget_scoped(const sdl_shape* shape, double sparsity, int scope) {
  if (scope == SDL_BUDGET_SEQUENCE) return sdl_mask_budget(shape, sparsity);
  if (scope != SDL_BUDGET_HEAD || check_shape(shape) != SDL_OK) return -1;
  if (!(sparsity >= 0.0 && sparsity < 1.0)) return -1;
  const int64_t nb = shape->L / shape->block;
  const int64_t kb = (int64_t)floor((1.0 - sparsity) * (double)nb * (double)nb + 0.5);
  if (kb < nb) return -1;
  return kb * shape->B * shape->H;
}

sdl_status sdl_block_scores(const void* q, const void* k, const sdl_shape* shape, float scale,
                            float* scores, void* workspace, size_t workspace_bytes,
                            void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (!q || !k || !scores) return SDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(scores)) return SDL_ERR_INVALID_ARG;
  if ((e = check_strides(s.q_strides, s.dtype, s.B, s.L, s.H)) ||
      (e = check_strides(s.k_strides, s.dtype, s.B, s.L, s.H_kv)))
    return e;
  const size_t need = sdl_scores_workspace_bytes(shape);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SDL_ERR_WORKSPACE;
  const size_t nb = s.L / s.block;
  float* qbar = static_cast<float*>(workspace);
  float* kbar = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         align256(sizeof(float) * s.B * s.H * nb * s.d));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t ce = launch_pool(q, k, s, qbar, kbar, st);
  if (ce != cudaSuccess) return cuda_fail(ce);
  ce = launch_scores(qbar, kbar, s, resolve_scale(scale, s.d), scores, st);
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_select_mask(const float* scores, const sdl_shape* shape, double sparsity,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                           uint8_t* mask_u8, void* workspace, size_t workspace_bytes,
                           void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!scores || !row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  if (!aligned16(scores)) return SDL_ERR_INVALID_ARG;
  const int64_t total = sdl_mask_budget(shape, sparsity);
  if (total < 0) return SDL_ERR_INVALID_ARG;
  if (col_capacity < total) return SDL_ERR_CAPACITY;
  const size_t need = sdl_select_workspace_bytes(shape);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SDL_ERR_WORKSPACE;
  const int nb = shape->L / shape->block;
  cudaError_t ce = launch_select(scores, shape->B, shape->H, nb, total / shape->B, row_ptr,
                                 col_idx, mask_u8, workspace, static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_select_mask_scoped(const float* scores, const sdl_shape* shape, double sparsity,
                                  int scope, int32_t* row_ptr, int32_t* col_idx,
                                  int64_t col_capacity, uint8_t* mask_u8, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (scope == SDL_BUDGET_SEQUENCE)
    return sdl_select_mask(scores, shape, sparsity, row_ptr, col_idx, col_capacity, mask_u8,
                           workspace, workspace_bytes, stream);
  if (scope != SDL_BUDGET_HEAD) return SDL_ERR_INVALID_ARG;
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!scores || !row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  if (!aligned16(scores)) return SDL_ERR_INVALID_ARG;
  const int64_t total = sdl_mask_budget_scoped(shape, sparsity, scope);
  if (total < 0) return SDL_ERR_INVALID_ARG;
  if (col_capacity < total) return SDL_ERR_CAPACITY;
  const size_t need = sdl_select_workspace_bytes_scoped(shape, scope);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SDL_ERR_WORKSPACE;
  const int nb = shape->L / shape->block;
  // every head is its own single-head sequence: same layouts, B*H sequences of H = 1
  const int seqs = shape->B * shape->H;
  cudaError_t ce = launch_select(scores, seqs, 1, nb, total / seqs, row_ptr, col_idx, mask_u8,
                                 workspace, static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

// ------------------------------------------------- fused anchor step

size_t sdl_anchor_workspace_bytes(const sdl_shape* shape) {
  if (check_shape(shape) != SDL_OK) return 0;
  return align256(sdl_scores_workspace_bytes(shape)) +
         align256(sdl_select_workspace_bytes(shape)) + anchor_barrier_bytes();
}

}  // extern "C"

namespace {

// Validation and workspace carving shared by the fused anchor entry points;
// `plan` is checked by the callers.
struct AnchorCall {
  float* qbar;
  float* kbar;
  char* sel;
  unsigned* bar;
  int* status;
  int64_t total;
};

sdl_status anchor_prepare(const void* q, const void* k, const sdl_shape* shape, double sparsity,
                          const float* scores, const int32_t* row_ptr, const int32_t* col_idx,
                          int64_t col_capacity, void* workspace, size_t workspace_bytes,
                          AnchorCall& c) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (!q || !k || !scores || !row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(scores)) return SDL_ERR_INVALID_ARG;
  if ((e = check_strides(s.q_strides, s.dtype, s.B, s.L, s.H)) ||
      (e = check_strides(s.k_strides, s.dtype, s.B, s.L, s.H_kv)))
    return e;
  c.total = sdl_mask_budget(shape, sparsity);
  if (c.total < 0) return SDL_ERR_INVALID_ARG;
  if (col_capacity < c.total) return SDL_ERR_CAPACITY;
  const size_t need = sdl_anchor_workspace_bytes(shape);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SDL_ERR_WORKSPACE;
  c.status = device_status_ptr();
  if (!c.status) return SDL_ERR_CUDA;
  const size_t nb = s.L / s.block;
  char* w = static_cast<char*>(workspace);
  c.qbar = reinterpret_cast<float*>(w);
  c.kbar = reinterpret_cast<float*>(w + align256(sizeof(float) * s.B * s.H * nb * s.d));
  c.sel = w + align256(sdl_scores_workspace_bytes(shape));
  c.bar = reinterpret_cast<unsigned*>(c.sel + align256(sdl_select_workspace_bytes(shape)));
  return SDL_OK;
}

}  // namespace

extern "C" {

sdl_status sdl_anchor_refresh(const void* q, const void* k, const sdl_shape* shape, float scale,
                              double sparsity, float* scores, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int32_t* plan,
                              void* workspace, size_t workspace_bytes, void* stream) {
  AnchorCall c;
  const sdl_status e = anchor_prepare(q, k, shape, sparsity, scores, row_ptr, col_idx,
                                      col_capacity, workspace, workspace_bytes, c);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (plan && s.block != 64) return SDL_ERR_INVALID_ARG;
  cudaError_t ce = launch_anchor(q, k, s, resolve_scale(scale, s.d), c.total / s.B, c.qbar,
                                 c.kbar, scores, c.sel, row_ptr, col_idx, plan, c.bar, c.status,
                                 static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_anchor_step(const void* q, const void* k, const sdl_shape* shape, float scale,
                           double sparsity, float* scores, int32_t* row_ptr, int32_t* col_idx,
                           int64_t col_capacity, int32_t* plan, int32_t* order, void* lists,
                           size_t lists_bytes, void* workspace, size_t workspace_bytes,
                           void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (s.block != 64) return SDL_ERR_UNSUPPORTED;
  if (!plan || !order) return SDL_ERR_INVALID_ARG;
  if (lists && !aligned16(lists)) return SDL_ERR_INVALID_ARG;
  if (lists && lists_bytes < sdl_tile_lists_bytes(shape)) return SDL_ERR_WORKSPACE;
  AnchorCall c;
  e = anchor_prepare(q, k, shape, sparsity, scores, row_ptr, col_idx, col_capacity, workspace,
                     workspace_bytes, c);
  if (e) return e;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nb = s.L / s.block;
  cudaError_t ce = launch_anchor(q, k, s, resolve_scale(scale, s.d), c.total / s.B, c.qbar,
                                 c.kbar, scores, c.sel, row_ptr, col_idx, nullptr, c.bar,
                                 c.status, st);
  if (ce == cudaSuccess) ce = launch_plan(row_ptr, col_idx, s.B, s.H, nb, plan, st);
  if (ce == cudaSuccess) ce = launch_tile_order(row_ptr, plan, s.B, s.H, nb, order, st);
  if (ce == cudaSuccess && lists)
    ce = launch_tile_lists(lists_args(s, row_ptr, col_idx, plan, order, c.status),
                           static_cast<int32_t*>(lists), st);
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

// ------------------------------------------------- column-sparse attention

int64_t sdl_col_budget(const sdl_shape* shape, double sparsity) {
  if (check_shape(shape) != SDL_OK) return -1;
  if (!(sparsity >= 0.0 && sparsity < 1.0)) return -1;
  int64_t c = 64 * (int64_t)floor((1.0 - sparsity) * (double)shape->L / 64.0 + 0.5);
  if (c < 64) c = 64;
  return c > shape->L ? shape->L : c;
}

size_t sdl_col_scores_workspace_bytes(const sdl_shape* shape) {
  if (check_shape(shape) != SDL_OK) return 0;
  const size_t nb = shape->L / shape->block;
  return align256(sdl_scores_workspace_bytes(shape)) +
         align256(sizeof(float) * 2 * shape->B * shape->H * nb) +
         align256(col_partial_bytes(*shape));
}

sdl_status sdl_col_scores(const void* q, const void* k, const sdl_shape* shape, float scale,
                          float* col_scores, void* workspace, size_t workspace_bytes,
                          void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (!q || !k || !col_scores) return SDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(col_scores)) return SDL_ERR_INVALID_ARG;
  if ((e = check_strides(s.q_strides, s.dtype, s.B, s.L, s.H)) ||
      (e = check_strides(s.k_strides, s.dtype, s.B, s.L, s.H_kv)))
    return e;
  const size_t need = sdl_col_scores_workspace_bytes(shape);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SDL_ERR_WORKSPACE;
  const size_t nb = s.L / s.block;
  char* w = static_cast<char*>(workspace);
  float* qbar = reinterpret_cast<float*>(w);
  float* kbar = reinterpret_cast<float*>(w + align256(sizeof(float) * s.B * s.H * nb * s.d));
  float2* stats = reinterpret_cast<float2*>(w + align256(sdl_scores_workspace_bytes(shape)));
  float2* part = reinterpret_cast<float2*>(w + align256(sdl_scores_workspace_bytes(shape)) +
                                           align256(sizeof(float) * 2 * s.B * s.H * nb));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t ce = launch_pool(q, k, s, qbar, kbar, st);
  if (ce != cudaSuccess) return cuda_fail(ce);
  ce = launch_col_scores(k, s, resolve_scale(scale, s.d), qbar, part, stats, col_scores, st);
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_col_select(const float* col_scores, const sdl_shape* shape, double sparsity,
                          int32_t* cols, int64_t col_capacity, void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!col_scores || !cols) return SDL_ERR_INVALID_ARG;
  const int64_t Lc = sdl_col_budget(shape, sparsity);
  if (Lc < 0) return SDL_ERR_INVALID_ARG;
  if (col_capacity < Lc * shape->B * shape->H) return SDL_ERR_CAPACITY;
  cudaError_t ce = launch_col_select(col_scores, shape->B * shape->H, shape->L, (int)Lc, cols,
                                     static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_col_gather(const void* k, const void* v, const sdl_shape* shape,
                          const int32_t* cols, int32_t Lc, void* k_cols, void* v_cols,
                          void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  const sdl_shape& s = *shape;
  if (!k || !v || !cols || !k_cols || !v_cols || Lc <= 0 || Lc > s.L) return SDL_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cols) || !aligned16(v_cols))
    return SDL_ERR_INVALID_ARG;
  if ((e = check_strides(s.k_strides, s.dtype, s.B, s.L, s.H_kv)) ||
      (e = check_strides(s.v_strides, s.dtype, s.B, s.L, s.H_kv)))
    return e;
  cudaError_t ce = launch_col_gather(k, v, s, cols, Lc, k_cols, v_cols,
                                     static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_col_sparse_attn(const void* q, const void* k_cols, const void* v_cols,
                               const sdl_shape* shape, int32_t Lc, float scale, void* o,
                               float* lse, void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (Lc <= 0 || Lc % 64 || Lc > shape->L) return SDL_ERR_INVALID_ARG;
  // the gathered tensors: one per query head, contiguous [B, Lc, H, d]
  sdl_shape loc = *shape;
  loc.H_kv = shape->H;
  const int64_t st[3] = {(int64_t)Lc * shape->H * shape->d, (int64_t)shape->H * shape->d,
                         (int64_t)shape->d};
  for (int i = 0; i < 3; ++i) loc.k_strides[i] = loc.v_strides[i] = st[i];
  return attn_common(q, k_cols, v_cols, &loc, nullptr, nullptr, nullptr, scale, o, lse, stream,
                     Lc);
}

// ------------------------------------------------- heads split over ranks

namespace {
// Free picks per sequence under the global budget of all `heads_total` heads
// (-1 if the arguments are invalid).
int64_t shard_kfree(const sdl_shape* local, int32_t heads_total, double sparsity) {
  if (check_shape(local) != SDL_OK) return -1;
  if (heads_total < local->H) return -1;
  if (!(sparsity >= 0.0 && sparsity < 1.0)) return -1;
  const int64_t nb = local->L / local->block;
  const int64_t kb =
      (int64_t)floor((1.0 - sparsity) * (double)heads_total * (double)nb * (double)nb + 0.5);
  const int64_t forced = (int64_t)heads_total * nb;
  if (kb < forced) return -1;
  return kb - forced;
}

sdl_status shard_args(const float* scores, const sdl_shape* local, int32_t heads_total,
                      double sparsity, void* workspace, size_t workspace_bytes, int64_t* kfree) {
  sdl_status e = check_shape(local);
  if (e) return e;
  *kfree = shard_kfree(local, heads_total, sparsity);
  if (*kfree < 0) return SDL_ERR_INVALID_ARG;
  if (!scores || !aligned16(scores)) return SDL_ERR_INVALID_ARG;
  const size_t need = sdl_select_shard_workspace_bytes(local);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SDL_ERR_WORKSPACE;
  return SDL_OK;
}
}  // namespace

size_t sdl_select_shard_workspace_bytes(const sdl_shape* local) {
  return sdl_select_workspace_bytes(local);
}

sdl_status sdl_select_shard_hist(const sdl_shape* local, int pass, size_t* offset_bytes,
                                 size_t* count) {
  sdl_status e = check_shape(local);
  if (e) return e;
  if (pass < 0 || pass >= SDL_SELECT_PASSES || !offset_bytes || !count) return SDL_ERR_INVALID_ARG;
  *offset_bytes = select_hist_offset(local->B, pass);
  *count = select_hist_count(local->B);
  return SDL_OK;
}

int64_t sdl_select_shard_capacity(const sdl_shape* local, int32_t heads_total, double sparsity) {
  const int64_t kfree = shard_kfree(local, heads_total, sparsity);
  if (kfree < 0) return -1;
  const int64_t nb = local->L / local->block;
  const int64_t rows = (int64_t)local->H * nb;
  const int64_t free_here = rows * (nb - 1) < kfree ? rows * (nb - 1) : kfree;
  return (rows + free_here) * local->B;
}

sdl_status sdl_select_shard_pass(const float* scores, const sdl_shape* local, int32_t heads_total,
                                 double sparsity, int pass, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  int64_t kfree = 0;
  sdl_status e = shard_args(scores, local, heads_total, sparsity, workspace, workspace_bytes, &kfree);
  if (e) return e;
  if (pass < 0 || pass >= SDL_SELECT_PASSES) return SDL_ERR_INVALID_ARG;
  cudaError_t ce = launch_select_shard_pass(scores, local->B, local->H, local->L / local->block,
                                            kfree, pass, workspace,
                                            static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_select_shard_count(const float* scores, const sdl_shape* local, int32_t heads_total,
                                  double sparsity, void* workspace, size_t workspace_bytes,
                                  int64_t* totals, void* stream) {
  int64_t kfree = 0;
  sdl_status e = shard_args(scores, local, heads_total, sparsity, workspace, workspace_bytes, &kfree);
  if (e) return e;
  if (!totals) return SDL_ERR_INVALID_ARG;
  cudaError_t ce = launch_select_shard_count(scores, local->B, local->H, local->L / local->block,
                                             kfree, workspace, totals,
                                             static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_select_shard_finish(const float* scores, const sdl_shape* local,
                                   int32_t heads_total, double sparsity, const int64_t* offsets,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   uint8_t* mask_u8, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  int64_t kfree = 0;
  sdl_status e = shard_args(scores, local, heads_total, sparsity, workspace, workspace_bytes, &kfree);
  if (e) return e;
  if (!offsets || !row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  if (col_capacity < sdl_select_shard_capacity(local, heads_total, sparsity))
    return SDL_ERR_CAPACITY;
  cudaError_t ce = launch_select_shard_finish(scores, local->B, local->H,
                                              local->L / local->block, kfree, offsets, workspace,
                                              row_ptr, col_idx, mask_u8,
                                              static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_sparse_attn(const void* q, const void* k, const void* v, const sdl_shape* shape,
                           const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                           float* lse, void* stream) {
  if (!row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  return attn_common(q, k, v, shape, row_ptr, col_idx, nullptr, scale, o, lse, stream);
}

sdl_status sdl_sparse_attn_planned(const void* q, const void* k, const void* v,
                                   const sdl_shape* shape, const int32_t* row_ptr,
                                   const int32_t* col_idx, const int32_t* plan, float scale,
                                   void* o, float* lse, void* stream) {
  if (!row_ptr || !col_idx) return SDL_ERR_INVALID_ARG;
  return attn_common(q, k, v, shape, row_ptr, col_idx, plan, scale, o, lse, stream);
}

sdl_status sdl_tile_plan(const int32_t* row_ptr, const int32_t* col_idx, const sdl_shape* shape,
                         int32_t* plan, void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!row_ptr || !col_idx || !plan) return SDL_ERR_INVALID_ARG;
  if (shape->block != 64) return SDL_ERR_UNSUPPORTED;
  const cudaError_t ce = launch_plan(row_ptr, col_idx, shape->B, shape->H,
                                     shape->L / shape->block, plan,
                                     static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_tile_order(const int32_t* row_ptr, const int32_t* plan, const sdl_shape* shape,
                          int32_t* order, void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!row_ptr || !plan || !order) return SDL_ERR_INVALID_ARG;
  if (shape->block != 64) return SDL_ERR_UNSUPPORTED;
  const cudaError_t ce = launch_tile_order(row_ptr, plan, shape->B, shape->H,
                                           shape->L / shape->block, order,
                                           static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_sparse_attn_scheduled(const void* q, const void* k, const void* v,
                                     const sdl_shape* shape, const int32_t* row_ptr,
                                     const int32_t* col_idx, const int32_t* plan,
                                     const int32_t* order, float scale, void* o, float* lse,
                                     void* stream) {
  if (!row_ptr || !col_idx || !plan || !order) return SDL_ERR_INVALID_ARG;
  return attn_common(q, k, v, shape, row_ptr, col_idx, plan, scale, o, lse, stream, 0, order);
}

size_t sdl_tile_lists_bytes(const sdl_shape* shape) {
  if (check_shape(shape) != SDL_OK) return 0;
  const int64_t n_items = (int64_t)shape->B * shape->H * ((shape->L + 127) / 128);
  return tile_lists_bytes(n_items, shape->L);
}

sdl_status sdl_tile_lists(const int32_t* row_ptr, const int32_t* col_idx, const int32_t* plan,
                          const int32_t* order, const sdl_shape* shape, void* lists,
                          size_t lists_bytes, void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!row_ptr || !col_idx || !lists || !aligned16(lists)) return SDL_ERR_INVALID_ARG;
  if (shape->block != 64) return SDL_ERR_UNSUPPORTED;
  if (lists_bytes < sdl_tile_lists_bytes(shape)) return SDL_ERR_WORKSPACE;
  int* status = device_status_ptr();
  if (!status) return SDL_ERR_CUDA;
  const AttnArgs a = lists_args(*shape, row_ptr, col_idx, plan, order, status);
  const cudaError_t ce =
      launch_tile_lists(a, static_cast<int32_t*>(lists), static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_sparse_attn_listed(const void* q, const void* k, const void* v,
                                  const sdl_shape* shape, const void* lists, float scale, void* o,
                                  float* lse, void* stream) {
  sdl_status e = check_shape(shape);
  if (e) return e;
  if (!lists || !aligned16(lists)) return SDL_ERR_INVALID_ARG;
  if (shape->block != 64 || shape->dtype != SDL_BF16) return SDL_ERR_UNSUPPORTED;
  return attn_common(q, k, v, shape, nullptr, nullptr, nullptr, scale, o, lse, stream, 0, nullptr,
                     static_cast<const int32_t*>(lists));
}

sdl_status sdl_dense_attn(const void* q, const void* k, const void* v, const sdl_shape* shape,
                          float scale, void* o, float* lse, void* stream) {
  return attn_common(q, k, v, shape, nullptr, nullptr, nullptr, scale, o, lse, stream);
}

sdl_status sdl_wait_selfcheck(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return SDL_ERR_INVALID_ARG;
  int* status = device_status_ptr();
  if (!status) return SDL_ERR_CUDA;
  cudaError_t ce = launch_wait_check(limit_ns, status, static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  return SDL_OK;
}

sdl_status sdl_last_device_status(void* stream) {
  cudaError_t ce = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce);
  int w[2] = {0, 0};
  ce = cudaMemcpyFromSymbol(w, g_device_status, sizeof(w));
  if (ce != cudaSuccess) return cuda_fail(ce);
  const int zero[2] = {0, 0};
  ce = cudaMemcpyToSymbol(g_device_status, zero, sizeof(zero));
  if (ce != cudaSuccess) return cuda_fail(ce);
  const int v = w[0];
  t_last_device_detail = (v & kDevBadMask) ? w[1] : 0;
  if (v & kDevTimeout) return SDL_ERR_TIMEOUT;
  if (v & kDevBadMask) return SDL_ERR_BAD_MASK;
  if (v & kDevOverlap) return SDL_ERR_OVERLAP;
  return SDL_OK;
}

int sdl_last_cuda_error(void) { return t_last_cuda_error; }

int sdl_last_device_detail(void) { return t_last_device_detail; }

const char* sdl_status_string(sdl_status status) {
  switch (status) {
    case SDL_OK:
      return "ok";
    case SDL_ERR_INVALID_ARG:
      return "invalid argument";
    case SDL_ERR_UNSUPPORTED:
      return "unsupported shape (d, block or L)";
    case SDL_ERR_CAPACITY:
      return "col_idx capacity below the mask budget";
    case SDL_ERR_WORKSPACE:
      return "workspace missing or too small";
    case SDL_ERR_CUDA:
      return "CUDA error (see sdl_last_cuda_error)";
    case SDL_ERR_TIMEOUT:
      return "a kernel's bounded wait timed out";
    case SDL_ERR_BAD_MASK:
      return "mask list entry out of range or out of order";
    case SDL_ERR_OVERLAP:
      return "attention launches in flight shared a tile counter";
  }
  return "unknown status";
}

}  // extern "C"
