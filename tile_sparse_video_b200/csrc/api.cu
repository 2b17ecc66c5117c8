// libvsa C ABI: argument checks, plan lifetime and dispatch to the kernels.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <new>
#include <string>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {

static thread_local std::string g_last_error;

// Bound of the attention kernels' mbarrier waits (process-wide; a test
// shortens it through vsa_debug_set_wait_limit to make the abort path run).
static std::atomic<unsigned long long> g_wait_limit_ns{sm100::kWaitLimitNs};

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(); }

void set_error(const std::string& msg) { g_last_error = msg; }

vsa_status fail(vsa_status code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

static vsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// Common checks for every launching call.  Returns VSA_OK and sets *empty when
// there is nothing to do (B*H == 0 or no tokens).
static vsa_status check_launch(const vsa_plan_s* p, int B, int H, int D, bool* empty) {
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (p->device < 0) return fail(VSA_ERR_INVALID_ARG, "host-only plan (device = -1) cannot launch");
  if (B < 0 || H < 0) return fail(VSA_ERR_INVALID_ARG, "B and H must be >= 0");
  if (D != 64 && D != 128) return fail(VSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != p->device)
    return fail(VSA_ERR_INVALID_ARG, "current CUDA device differs from the plan's device");
  *empty = (int64_t(B) * H == 0) || p->n_tokens == 0;
  return VSA_OK;
}

static vsa_status check_ptr(const void* ptr, const char* name) {
  if (ptr == nullptr) return fail(VSA_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!aligned16(ptr)) return fail(VSA_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  return VSA_OK;
}

static vsa_status check_k(const vsa_plan_s* p, int k) {
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  if (k < 0 || k > n_v) return fail(VSA_ERR_INVALID_ARG, "k must be in [0, n_video_tiles]");
  if (k == 0 && p->n_prefix_tiles == 0 && n_v > 0)
    return fail(VSA_ERR_INVALID_ARG, "k = 0 without prefix tiles leaves no key to attend to");
  return VSA_OK;
}

#define VSA_TRY(expr)                 \
  do {                                \
    vsa_status _s = (expr);           \
    if (_s != VSA_OK) return _s;      \
  } while (0)

}  // namespace vsa

using namespace vsa;

extern "C" {

const char* vsa_last_error(void) { return g_last_error.c_str(); }

vsa_status vsa_plan_create(const vsa_geometry* geom, int device, vsa_plan* out) {
  if (geom == nullptr || out == nullptr) return fail(VSA_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  vsa_plan_s* p = new (std::nothrow) vsa_plan_s();
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "out of host memory");
  vsa_status st = build_plan(*geom, p);
  if (st != VSA_OK) {
    delete p;
    return st;
  }
  if (device >= 0) {
    int prev = -1;
    cudaError_t e = cudaGetDevice(&prev);
    if (e == cudaSuccess) e = cudaSetDevice(device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, device);
    const size_t nb_u = sizeof(int32_t) * std::max<size_t>(1, p->untile.size());
    const size_t nb_r = sizeof(int32_t) * std::max<size_t>(1, p->row_src.size());
    const size_t nb_b = sizeof(int32_t) * std::max<size_t>(1, p->block_len.size());
    if (e == cudaSuccess) e = cudaMalloc(&p->d_untile, nb_u);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_row_src, nb_r);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_block_len, nb_b);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_status, 32);
    if (e == cudaSuccess && !p->untile.empty())
      e = cudaMemcpy(p->d_untile, p->untile.data(), p->untile.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !p->row_src.empty())
      e = cudaMemcpy(p->d_row_src, p->row_src.data(), p->row_src.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !p->block_len.empty())
      e = cudaMemcpy(p->d_block_len, p->block_len.data(), p->block_len.size() * 4,
                     cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, 32);
    if (prev >= 0) cudaSetDevice(prev);
    if (e != cudaSuccess) {
      p->device = device;
      vsa_plan_destroy(p);
      return cuda_fail(e, "uploading plan tables");
    }
    p->device = device;
  }
  *out = p;
  return VSA_OK;
}

vsa_status vsa_plan_info(vsa_plan p, int64_t* n_tokens, int64_t* n_padded, int32_t* n_tiles,
                         int32_t* n_prefix_tiles, int32_t* tile_rows) {
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (n_tokens) *n_tokens = p->n_tokens;
  if (n_padded) *n_padded = p->n_padded;
  if (n_tiles) *n_tiles = p->n_tiles;
  if (n_prefix_tiles) *n_prefix_tiles = p->n_prefix_tiles;
  if (tile_rows) *tile_rows = p->R;
  return VSA_OK;
}

vsa_status vsa_plan_tables(vsa_plan p, int32_t* untile, int32_t* row_src, int32_t* block_len,
                           int32_t* tile_seg) {
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (untile) std::copy(p->untile.begin(), p->untile.end(), untile);
  if (row_src) std::copy(p->row_src.begin(), p->row_src.end(), row_src);
  if (block_len) std::copy(p->block_len.begin(), p->block_len.end(), block_len);
  if (tile_seg) std::copy(p->tile_seg.begin(), p->tile_seg.end(), tile_seg);
  return VSA_OK;
}

vsa_status vsa_keep_count(vsa_plan p, double keep_ratio, int32_t keep_tiles, int32_t* k) {
  if (p == nullptr || k == nullptr) return fail(VSA_ERR_INVALID_ARG, "NULL argument");
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  int64_t kk;
  if (keep_tiles >= 0) {
    kk = std::min<int64_t>(keep_tiles, n_v);
  } else {
    if (!(keep_ratio == keep_ratio)) return fail(VSA_ERR_INVALID_ARG, "keep_ratio is NaN");
    const double r = std::min(1.0, std::max(0.0, keep_ratio));
    kk = std::min<int64_t>(n_v, int64_t(std::ceil(r * n_v - 1e-9)));
    kk = std::max<int64_t>(kk, 0);
  }
  if (kk == 0 && p->n_prefix_tiles == 0 && n_v > 0)
    return fail(VSA_ERR_INVALID_ARG, "k = 0 without prefix tiles leaves no key to attend to");
  *k = int32_t(kk);
  return VSA_OK;
}

vsa_status vsa_plan_destroy(vsa_plan p) {
  if (p == nullptr) return VSA_OK;
  if (p->device >= 0) {
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(p->device);
    cudaFree(p->d_untile);
    cudaFree(p->d_row_src);
    cudaFree(p->d_block_len);
    cudaFree(p->d_status);
    if (prev >= 0) cudaSetDevice(prev);
  }
  delete p;
  return VSA_OK;
}

vsa_status vsa_workspace_size(vsa_plan p, int B, int H, int D, int k, size_t* bytes) {
  if (p == nullptr || bytes == nullptr) return fail(VSA_ERR_INVALID_ARG, "NULL argument");
  if (B < 0 || H < 0) return fail(VSA_ERR_INVALID_ARG, "B and H must be >= 0");
  if (D != 64 && D != 128) return fail(VSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128");
  (void)k;
  // the pooled means, then the coarse kernel's score rows
  *bytes = size_t(3) * size_t(B) * size_t(H) * size_t(p->n_tiles) * size_t(D) * sizeof(float) +
           coarse_scratch_bytes(p->n_tiles, p->num_sms);
  return VSA_OK;
}

vsa_status vsa_permute(vsa_plan p, const void* x, void* x_t, int B, int H, int D, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(x, "x"));
  VSA_TRY(check_ptr(x_t, "x_t"));
  cudaError_t e = launch_gather_rows(static_cast<const uint16_t*>(x), static_cast<uint16_t*>(x_t),
                                     p->d_row_src, int64_t(B) * H, p->n_tokens, p->n_padded, D,
                                     p->num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "vsa_permute launch");
}

vsa_status vsa_unpermute(vsa_plan p, const void* x_t, void* x, int B, int H, int D, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(x_t, "x_t"));
  VSA_TRY(check_ptr(x, "x"));
  cudaError_t e = launch_gather_rows(static_cast<const uint16_t*>(x_t), static_cast<uint16_t*>(x),
                                     p->d_untile, int64_t(B) * H, p->n_padded, p->n_tokens, D,
                                     p->num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "vsa_unpermute launch");
}

vsa_status vsa_coarse_topk(vsa_plan p, const void* q_t, const void* k_t, const void* v_t, int B,
                           int H, int D, float scale, int k, float* o_coarse, int32_t* topk_idx,
                           float* topk_score, void* ws, size_t ws_bytes, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  VSA_TRY(check_k(p, k));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(q_t, "q_t"));
  VSA_TRY(check_ptr(k_t, "k_t"));
  VSA_TRY(check_ptr(v_t, "v_t"));
  VSA_TRY(check_ptr(o_coarse, "o_coarse"));
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  if (k > 0 && n_v > 0) VSA_TRY(check_ptr(topk_idx, "topk_idx"));
  if (topk_score != nullptr && !aligned16(topk_score))
    return fail(VSA_ERR_INVALID_ARG, "topk_score is not 16-byte aligned");
  if (!std::isfinite(scale)) return fail(VSA_ERR_INVALID_ARG, "scale is not finite");
  if (p->n_tiles > 4096)
    return fail(VSA_ERR_UNSUPPORTED, "coarse attention supports at most 4096 tiles");
  size_t need = 0;
  vsa_workspace_size(p, B, H, D, k, &need);
  if (ws == nullptr || ws_bytes < need)
    return fail(VSA_ERR_WORKSPACE, "workspace missing or too small (see vsa_workspace_size)");
  if (!aligned16(ws)) return fail(VSA_ERR_INVALID_ARG, "ws is not 16-byte aligned");
  const int64_t bh = int64_t(B) * H;
  float* qbar = static_cast<float*>(ws);
  float* kbar = qbar + bh * p->n_tiles * D;
  float* vbar = kbar + bh * p->n_tiles * D;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_pool(static_cast<const uint16_t*>(q_t), static_cast<const uint16_t*>(k_t),
                              static_cast<const uint16_t*>(v_t), p->d_block_len, qbar, kbar, vbar,
                              bh, p->n_tiles, p->R, D, p->num_sms, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool launch");
  float* scratch = qbar + size_t(3) * bh * p->n_tiles * D;
  e = launch_coarse_topk(qbar, kbar, vbar, bh, p->n_tiles, p->n_prefix_tiles, D, scale, k,
                         o_coarse, topk_idx, topk_score, scratch, p->num_sms, s);
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "coarse_topk launch");
}

vsa_status vsa_permute_pool(vsa_plan p, const void* x, void* x_t, int B, int H, int D,
                            float* pooled, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(x, "x"));
  VSA_TRY(check_ptr(x_t, "x_t"));
  VSA_TRY(check_ptr(pooled, "pooled"));
  cudaError_t e = launch_permute_pool(static_cast<const uint16_t*>(x), static_cast<uint16_t*>(x_t),
                                      p->d_row_src, p->d_block_len, pooled, int64_t(B) * H,
                                      p->n_tiles, p->R, p->n_tokens, p->n_padded, D, p->num_sms,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "vsa_permute_pool launch");
}

vsa_status vsa_coarse_topk_pooled(vsa_plan p, int B, int H, int D, float scale, int k,
                                  float* o_coarse, int32_t* topk_idx, float* topk_score, void* ws,
                                  size_t ws_bytes, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  VSA_TRY(check_k(p, k));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(o_coarse, "o_coarse"));
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  if (k > 0 && n_v > 0) VSA_TRY(check_ptr(topk_idx, "topk_idx"));
  if (topk_score != nullptr && !aligned16(topk_score))
    return fail(VSA_ERR_INVALID_ARG, "topk_score is not 16-byte aligned");
  if (!std::isfinite(scale)) return fail(VSA_ERR_INVALID_ARG, "scale is not finite");
  if (p->n_tiles > 4096)
    return fail(VSA_ERR_UNSUPPORTED, "coarse attention supports at most 4096 tiles");
  size_t need = 0;
  vsa_workspace_size(p, B, H, D, k, &need);
  if (ws == nullptr || ws_bytes < need)
    return fail(VSA_ERR_WORKSPACE, "workspace missing or too small (see vsa_workspace_size)");
  if (!aligned16(ws)) return fail(VSA_ERR_INVALID_ARG, "ws is not 16-byte aligned");
  const int64_t bh = int64_t(B) * H;
  const float* qbar = static_cast<const float*>(ws);
  const float* kbar = qbar + bh * p->n_tiles * D;
  const float* vbar = kbar + bh * p->n_tiles * D;
  float* scratch = const_cast<float*>(qbar) + size_t(3) * bh * p->n_tiles * D;
  cudaError_t e = launch_coarse_topk(qbar, kbar, vbar, bh, p->n_tiles, p->n_prefix_tiles, D, scale,
                                     k, o_coarse, topk_idx, topk_score, scratch, p->num_sms,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "coarse_topk launch");
}

vsa_status vsa_project(vsa_plan p, const void* x, const void* w, int B, int H, int D, int C,
                       int act, void* y, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (C <= 0 || C % 8 != 0) return fail(VSA_ERR_INVALID_ARG, "C must be a positive multiple of 8");
  if (act != 0 && act != 1) return fail(VSA_ERR_INVALID_ARG, "act must be 0 (identity) or 1 (sigmoid)");
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(x, "x"));
  VSA_TRY(check_ptr(w, "w"));
  VSA_TRY(check_ptr(y, "y"));
  return launch_project(p, x, w, B, H, D, C, act, 0, y, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_project_tiled(vsa_plan p, const void* x_t, const void* w, int B, int H, int D, int C,
                             int act, void* y_t, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (C <= 0 || C % 8 != 0) return fail(VSA_ERR_INVALID_ARG, "C must be a positive multiple of 8");
  if (act != 0 && act != 1) return fail(VSA_ERR_INVALID_ARG, "act must be 0 (identity) or 1 (sigmoid)");
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(x_t, "x_t"));
  VSA_TRY(check_ptr(w, "w"));
  VSA_TRY(check_ptr(y_t, "y_t"));
  return launch_project(p, x_t, w, B, H, D, C, act, 1, y_t, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_permute_rows(vsa_plan p, const void* x, void* x_t, int B, int C, void* stream) {
  VSA_NVTX_RANGE();
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (p->device < 0) return fail(VSA_ERR_INVALID_ARG, "host-only plan (device = -1) cannot launch");
  if (B < 0) return fail(VSA_ERR_INVALID_ARG, "B must be >= 0");
  if (C <= 0 || C % 8 != 0) return fail(VSA_ERR_INVALID_ARG, "C must be a positive multiple of 8");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != p->device)
    return fail(VSA_ERR_INVALID_ARG, "current CUDA device differs from the plan's device");
  if (B == 0 || p->n_tokens == 0) return VSA_OK;
  VSA_TRY(check_ptr(x, "x"));
  VSA_TRY(check_ptr(x_t, "x_t"));
  e = launch_gather_wide(static_cast<const uint16_t*>(x), static_cast<uint16_t*>(x_t), p->d_row_src,
                         B, p->n_tokens, p->n_padded, C, p->num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "permute_rows launch");
}

vsa_status vsa_sparse_attn(vsa_plan p, const void* q_t, const void* k_t, const void* v_t,
                           const int32_t* topk_idx, int B, int H, int D, int k, float scale,
                           void* o_fine_t, float* lse_t, void* ws, size_t ws_bytes,
                           void* stream) {
  VSA_NVTX_RANGE();
  (void)ws;
  (void)ws_bytes;
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  VSA_TRY(check_k(p, k));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(q_t, "q_t"));
  VSA_TRY(check_ptr(k_t, "k_t"));
  VSA_TRY(check_ptr(v_t, "v_t"));
  VSA_TRY(check_ptr(o_fine_t, "o_fine_t"));
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  if (k > 0 && n_v > 0) VSA_TRY(check_ptr(topk_idx, "topk_idx"));
  if (lse_t != nullptr && !aligned16(lse_t))
    return fail(VSA_ERR_INVALID_ARG, "lse_t is not 16-byte aligned");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  return launch_sparse_attn(p, q_t, k_t, v_t, topk_idx, int64_t(B) * H, D, k, scale, o_fine_t,
                            lse_t, nullptr, nullptr, nullptr, -1, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_sparse_attn_combine(vsa_plan p, const void* q_t, const void* k_t, const void* v_t,
                                   const int32_t* topk_idx, int B, int H, int D, int k, float scale,
                                   const void* gate, const float* o_coarse, void* out,
                                   float* lse_t, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  VSA_TRY(check_k(p, k));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(q_t, "q_t"));
  VSA_TRY(check_ptr(k_t, "k_t"));
  VSA_TRY(check_ptr(v_t, "v_t"));
  VSA_TRY(check_ptr(gate, "gate"));
  VSA_TRY(check_ptr(o_coarse, "o_coarse"));
  VSA_TRY(check_ptr(out, "out"));
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  if (k > 0 && n_v > 0) VSA_TRY(check_ptr(topk_idx, "topk_idx"));
  if (lse_t != nullptr && !aligned16(lse_t))
    return fail(VSA_ERR_INVALID_ARG, "lse_t is not 16-byte aligned");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  return launch_sparse_attn(p, q_t, k_t, v_t, topk_idx, int64_t(B) * H, D, k, scale, out, lse_t,
                            gate, o_coarse, nullptr, -1, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_keep_count_ref(vsa_plan p, double keep_ratio, int32_t keep_tiles, int32_t* k_ref) {
  if (p == nullptr || k_ref == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan or k_ref is NULL");
  const int n_p = p->n_prefix_tiles;
  int64_t kk = 0;
  if (keep_tiles >= 0) {
    kk = std::min<int64_t>(keep_tiles, n_p);
  } else {
    if (!(keep_ratio == keep_ratio)) return fail(VSA_ERR_INVALID_ARG, "keep_ratio is NaN");
    const double r = std::min(1.0, std::max(0.0, keep_ratio));
    kk = std::min<int64_t>(n_p, int64_t(std::ceil(r * n_p - 1e-9)));
  }
  *k_ref = int32_t(kk);
  return VSA_OK;
}

vsa_status vsa_select_reference(vsa_plan p, int B, int H, int D, float scale, int k_ref,
                                int32_t* topk_ref_idx, const void* ws, size_t ws_bytes,
                                void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (k_ref < 0 || k_ref > p->n_prefix_tiles)
    return fail(VSA_ERR_INVALID_ARG, "k_ref must be in [0, n_prefix_tiles]");
  if (p->n_prefix_tiles > 256)
    return fail(VSA_ERR_UNSUPPORTED, "reference selection supports at most 256 prefix tiles");
  if (empty || k_ref == 0 || p->n_tiles == p->n_prefix_tiles) return VSA_OK;
  VSA_TRY(check_ptr(topk_ref_idx, "topk_ref_idx"));
  if (!std::isfinite(scale)) return fail(VSA_ERR_INVALID_ARG, "scale is not finite");
  size_t need = 0;
  vsa_workspace_size(p, B, H, D, 0, &need);
  if (ws == nullptr || ws_bytes < need)
    return fail(VSA_ERR_WORKSPACE, "workspace missing or too small (see vsa_workspace_size)");
  if (!aligned16(ws)) return fail(VSA_ERR_INVALID_ARG, "ws is not 16-byte aligned");
  const int64_t bh = int64_t(B) * H;
  const float* qbar = static_cast<const float*>(ws);
  const float* kbar = qbar + bh * p->n_tiles * D;
  cudaError_t e = launch_select_ref(qbar, kbar, bh, p->n_tiles, p->n_prefix_tiles, D, scale, k_ref,
                                    topk_ref_idx, p->num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "select_ref launch");
}

vsa_status vsa_sparse_attn_ref(vsa_plan p, const void* q_t, const void* k_t, const void* v_t,
                               const int32_t* topk_idx, int k, const int32_t* topk_ref_idx,
                               int k_ref, int B, int H, int D, float scale, const void* gate,
                               const float* o_coarse, void* out, float* lse_t, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  const int n_p = p->n_prefix_tiles, n_v = p->n_tiles - p->n_prefix_tiles;
  if (k < 0 || k > n_v) return fail(VSA_ERR_INVALID_ARG, "k must be in [0, n_video_tiles]");
  if (k_ref < 0 || k_ref > n_p) return fail(VSA_ERR_INVALID_ARG, "k_ref must be in [0, n_prefix_tiles]");
  if (n_v > 0 && k + k_ref == 0)
    return fail(VSA_ERR_INVALID_ARG, "k + k_ref must be >= 1 (a video query tile needs a key)");
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(q_t, "q_t"));
  VSA_TRY(check_ptr(k_t, "k_t"));
  VSA_TRY(check_ptr(v_t, "v_t"));
  VSA_TRY(check_ptr(out, "out"));
  if (k > 0 && n_v > 0) VSA_TRY(check_ptr(topk_idx, "topk_idx"));
  // k_ref = n_p with no list: every reference tile, the unthinned layer
  const bool all_refs = k_ref == n_p && topk_ref_idx == nullptr;
  if (k_ref > 0 && n_v > 0 && !all_refs) VSA_TRY(check_ptr(topk_ref_idx, "topk_ref_idx"));
  if ((gate == nullptr) != (o_coarse == nullptr))
    return fail(VSA_ERR_INVALID_ARG, "gate and o_coarse are given together or not at all");
  if (gate != nullptr) {
    VSA_TRY(check_ptr(gate, "gate"));
    VSA_TRY(check_ptr(o_coarse, "o_coarse"));
  }
  if (lse_t != nullptr && !aligned16(lse_t))
    return fail(VSA_ERR_INVALID_ARG, "lse_t is not 16-byte aligned");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  return launch_sparse_attn(p, q_t, k_t, v_t, topk_idx, int64_t(B) * H, D, k, scale, out, lse_t,
                            gate, o_coarse, all_refs ? nullptr : topk_ref_idx, all_refs ? -1 : k_ref,
                            static_cast<cudaStream_t>(stream));
}

vsa_status vsa_gate_combine(vsa_plan p, const void* o_fine_t, const void* gate_t,
                            const float* o_coarse, void* out, int out_natural, int B, int H,
                            int D, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(o_fine_t, "o_fine_t"));
  VSA_TRY(check_ptr(gate_t, "gate_t"));
  VSA_TRY(check_ptr(o_coarse, "o_coarse"));
  VSA_TRY(check_ptr(out, "out"));
  if (out_natural != 0 && out_natural != 1)
    return fail(VSA_ERR_INVALID_ARG, "out_natural must be 0 or 1");
  cudaError_t e = launch_gate_combine(
      static_cast<const uint16_t*>(o_fine_t), static_cast<const uint16_t*>(gate_t), o_coarse,
      static_cast<uint16_t*>(out), out_natural, p->d_row_src, p->d_untile, int64_t(B) * H,
      p->n_tokens, p->n_padded, p->R, p->n_tiles, D, p->num_sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "gate_combine launch");
}

vsa_status vsa_backward_workspace_size(vsa_plan p, int B, int H, int D, size_t* bytes) {
  if (p == nullptr || bytes == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan or bytes is NULL");
  if (B < 0 || H < 0) return fail(VSA_ERR_INVALID_ARG, "B and H must be >= 0");
  if (D != 64 && D != 128) return fail(VSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128");
  const int64_t bh = int64_t(B) * H;
  *bytes = std::max(colmask_bytes(p, bh), coarse_bwd_bytes(p, bh));
  return VSA_OK;
}

vsa_status vsa_combine_backward(vsa_plan p, const void* d_out_t, const void* o_fine_t,
                                const void* gate_t, const float* o_coarse, int B, int H, int D,
                                float* delta, void* d_gate_t, float* d_o_coarse, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(d_out_t, "d_out_t"));
  VSA_TRY(check_ptr(o_fine_t, "o_fine_t"));
  VSA_TRY(check_ptr(gate_t, "gate_t"));
  VSA_TRY(check_ptr(o_coarse, "o_coarse"));
  VSA_TRY(check_ptr(delta, "delta"));
  VSA_TRY(check_ptr(d_gate_t, "d_gate_t"));
  VSA_TRY(check_ptr(d_o_coarse, "d_o_coarse"));
  cudaError_t e = launch_combine_backward(p, d_out_t, o_fine_t, gate_t, o_coarse, int64_t(B) * H, D,
                                          delta, d_gate_t, d_o_coarse,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "combine backward launch");
}

vsa_status vsa_coarse_backward(vsa_plan p, const float* qbar, const float* kbar, const float* vbar,
                               const float* d_o_coarse, int B, int H, int D, float scale,
                               float* d_qbar, float* d_kbar, float* d_vbar, void* ws,
                               size_t ws_bytes, void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(qbar, "qbar"));
  VSA_TRY(check_ptr(kbar, "kbar"));
  VSA_TRY(check_ptr(vbar, "vbar"));
  VSA_TRY(check_ptr(d_o_coarse, "d_o_coarse"));
  VSA_TRY(check_ptr(d_qbar, "d_qbar"));
  VSA_TRY(check_ptr(d_kbar, "d_kbar"));
  VSA_TRY(check_ptr(d_vbar, "d_vbar"));
  VSA_TRY(check_ptr(ws, "ws"));
  if (ws_bytes < coarse_bwd_bytes(p, int64_t(B) * H))
    return fail(VSA_ERR_WORKSPACE, "workspace smaller than vsa_backward_workspace_size");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  cudaError_t e = launch_coarse_backward(p, qbar, kbar, vbar, d_o_coarse, int64_t(B) * H, D, scale,
                                         d_qbar, d_kbar, d_vbar, ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "coarse backward launch");
}

vsa_status vsa_sparse_attn_backward(vsa_plan p, const void* q_t, const void* k_t, const void* v_t,
                                    const void* d_out_t, const int32_t* topk_idx, int k,
                                    const int32_t* topk_ref_idx, int k_ref, const float* lse_t,
                                    const float* delta, const float* d_qbar, const float* d_kbar,
                                    const float* d_vbar, int B, int H, int D, float scale,
                                    void* dq_t, void* dk_t, void* dv_t, void* ws, size_t ws_bytes,
                                    void* stream) {
  VSA_NVTX_RANGE();
  bool empty = false;
  VSA_TRY(check_launch(p, B, H, D, &empty));
  const int n_p = p->n_prefix_tiles, n_v = p->n_tiles - p->n_prefix_tiles;
  if (k < 0 || k > n_v) return fail(VSA_ERR_INVALID_ARG, "k must be in [0, n_video_tiles]");
  if (k_ref < 0 || k_ref > n_p) return fail(VSA_ERR_INVALID_ARG, "k_ref must be in [0, n_prefix_tiles]");
  if (n_v > 0 && k + k_ref == 0)
    return fail(VSA_ERR_INVALID_ARG, "k + k_ref must be >= 1 (a video query tile needs a key)");
  if (empty) return VSA_OK;
  VSA_TRY(check_ptr(q_t, "q_t"));
  VSA_TRY(check_ptr(k_t, "k_t"));
  VSA_TRY(check_ptr(v_t, "v_t"));
  VSA_TRY(check_ptr(d_out_t, "d_out_t"));
  VSA_TRY(check_ptr(lse_t, "lse_t"));
  VSA_TRY(check_ptr(delta, "delta"));
  VSA_TRY(check_ptr(dq_t, "dq_t"));
  VSA_TRY(check_ptr(dk_t, "dk_t"));
  VSA_TRY(check_ptr(dv_t, "dv_t"));
  VSA_TRY(check_ptr(ws, "ws"));
  if (k > 0 && n_v > 0) VSA_TRY(check_ptr(topk_idx, "topk_idx"));
  const bool all_refs = k_ref == n_p && topk_ref_idx == nullptr;
  if (k_ref > 0 && n_v > 0 && !all_refs) VSA_TRY(check_ptr(topk_ref_idx, "topk_ref_idx"));
  const int given = (d_qbar != nullptr) + (d_kbar != nullptr) + (d_vbar != nullptr);
  if (given != 0 && given != 3)
    return fail(VSA_ERR_INVALID_ARG, "d_qbar, d_kbar and d_vbar are given together or not at all");
  if (given == 3) {
    VSA_TRY(check_ptr(d_qbar, "d_qbar"));
    VSA_TRY(check_ptr(d_kbar, "d_kbar"));
    VSA_TRY(check_ptr(d_vbar, "d_vbar"));
  }
  if (ws_bytes < colmask_bytes(p, int64_t(B) * H))
    return fail(VSA_ERR_WORKSPACE, "workspace smaller than vsa_backward_workspace_size");
  if (!(scale > 0.0f) || !std::isfinite(scale))
    return fail(VSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  return launch_sparse_attn_backward(p, q_t, k_t, v_t, d_out_t, topk_idx, k,
                                     all_refs ? nullptr : topk_ref_idx, all_refs ? -1 : k_ref,
                                     lse_t, delta, d_qbar, d_kbar, d_vbar, int64_t(B) * H, D, scale,
                                     dq_t, dk_t, dv_t, ws, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_check_bounded_wait(vsa_plan p, int32_t* result, void* stream) {
  VSA_NVTX_RANGE();
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (p->device < 0) return fail(VSA_ERR_INVALID_ARG, "host-only plan (device = -1) cannot launch");
  VSA_TRY(check_ptr(result, "result"));
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != p->device)
    return fail(VSA_ERR_INVALID_ARG, "current CUDA device differs from the plan's device");
  e = launch_bounded_wait_check(p->d_status, reinterpret_cast<int*>(result),
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "bounded-wait check launch");
}

vsa_status vsa_debug_set_wait_limit(uint64_t ns) {
  // 0 restores the default; anything above the default is capped to it
  const unsigned long long lim =
      (ns == 0 || ns > sm100::kWaitLimitNs) ? sm100::kWaitLimitNs : (unsigned long long)ns;
  g_wait_limit_ns.store(lim);
  return VSA_OK;
}

vsa_status vsa_sync_status(vsa_plan p, void* stream) {
  VSA_NVTX_RANGE();
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (p->device < 0) return VSA_OK;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int st[4] = {0, 0, 0, 0};
  e = cudaMemcpy(st, p->d_status, sizeof(st), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, sizeof(st));
  if (e != cudaSuccess) return cuda_fail(e, "reading device status");
  if (st[0] == kStatusTimeout)
    return fail(VSA_ERR_DEVICE_TIMEOUT, "a kernel wait exceeded its bound (code " +
                                            std::to_string(st[1]) + ")");
  if (st[0] == kStatusBadIndex)
    return fail(VSA_ERR_DEVICE_INDEX, "a kept-tile index was outside [n_p, T) (value " +
                                          std::to_string(int(st[1])) + ")");
  return VSA_OK;
}

}  // extern "C"
