// Internal declarations shared by the libvsa translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/vsa.h"

struct vsa_plan_s {
  // geometry
  int R = 0;                 // rows per tile
  int64_t n_tokens = 0;      // N
  int64_t n_padded = 0;      // N_pad = T * R
  int n_tiles = 0;           // T
  int n_prefix_tiles = 0;    // n_p
  // host tables
  std::vector<int32_t> untile, row_src, block_len, tile_seg;
  // device side (device < 0: host-only plan)
  int device = -1;
  int num_sms = 0;
  int32_t* d_untile = nullptr;
  int32_t* d_row_src = nullptr;
  int32_t* d_block_len = nullptr;
  // device status word (0 = ok) in [0, 4); [4, 6): the attention kernel's
  // work counter (next item, CTAs done), zero between launches
  unsigned int* d_status = nullptr;
};

namespace vsa {

// An NVTX range named after the entry point around each call that launches
// work, so that a profiler's timeline (and ncu's --nvtx filters) show the
// library's calls.  NVTX is header-only and does nothing unless a tool is
// attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define VSA_NVTX_RANGE() ::vsa::NvtxRange vsa_nvtx_range_(__func__)

// Bound of the attention kernels' mbarrier waits, in ns (2 s unless a test
// shortened it through vsa_debug_set_wait_limit).
unsigned long long wait_limit_ns();

// Thread-local last error message.
void set_error(const std::string& msg);
vsa_status fail(vsa_status code, const std::string& msg);

// Host planner (plan.cpp).  Fills tables and sizes; returns VSA_OK or VSA_ERR_PLAN.
vsa_status build_plan(const vsa_geometry& g, vsa_plan_s* p);

// Kernel launchers (each .cu file); all asynchronous on `stream`.
cudaError_t launch_gather_rows(const uint16_t* src, uint16_t* dst, const int32_t* map,
                               int64_t bh, int64_t src_rows, int64_t dst_rows, int D,
                               int num_sms, cudaStream_t stream);
// Rows of C bf16 (C a multiple of 8): dst[b, r] = map[r] >= 0 ? src[b, map[r]] : 0.
cudaError_t launch_gather_wide(const uint16_t* src, uint16_t* dst, const int32_t* map, int64_t B,
                               int64_t src_rows, int64_t dst_rows, int C, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_pool(const uint16_t* q_t, const uint16_t* k_t, const uint16_t* v_t,
                        const int32_t* block_len, float* qbar, float* kbar, float* vbar,
                        int64_t bh, int T, int R, int D, int num_sms, cudaStream_t stream);
cudaError_t launch_permute_pool(const uint16_t* src, uint16_t* dst, const int32_t* row_src,
                                const int32_t* block_len, float* pooled, int64_t bh, int T, int R,
                                int64_t src_rows, int64_t dst_rows, int D, int num_sms,
                                cudaStream_t stream);
// Score rows of the coarse kernel's persistent CTAs (global scratch, bytes).
size_t coarse_scratch_bytes(int T, int num_sms);
cudaError_t launch_coarse_topk(const float* qbar, const float* kbar, const float* vbar,
                               int64_t bh, int T, int n_p, int D, float scale, int k,
                               float* o_coarse, int32_t* topk_idx, float* topk_score,
                               float* scratch, int num_sms, cudaStream_t stream);
// Top k_ref reference tiles per video query tile (n_p <= 256), ascending.
cudaError_t launch_select_ref(const float* qbar, const float* kbar, int64_t bh, int T, int n_p, int D,
                              float scale, int k_ref, int32_t* topk_ref, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_gate_combine(const uint16_t* o_fine_t, const uint16_t* gate_t,
                                const float* o_coarse, uint16_t* out, int out_natural,
                                const int32_t* row_src, const int32_t* untile,
                                int64_t bh, int64_t n_tokens, int64_t n_padded, int R, int T,
                                int D, int num_sms, cudaStream_t stream);
// gate == nullptr: o_fine in the padded layout; otherwise the fused gated
// combine writing natural order (gate natural [BH,N,D], o_coarse [BH,T,D]).
// k_ref < 0: every reference tile is a key of every video query tile;
// otherwise only its k_ref kept reference tiles, topk_ref [BH,n_v,k_ref].
vsa_status launch_sparse_attn(const vsa_plan_s* p, const void* q_t, const void* k_t,
                              const void* v_t, const int32_t* topk_idx, int64_t bh, int D,
                              int k, float scale, void* out, float* lse_t, const void* gate,
                              const float* o_coarse, const int32_t* topk_ref, int k_ref,
                              cudaStream_t stream);

// tiled = 0: x [B, N, C] natural rows -> y [B, H, N, D]; tiled = 1: x [B, N_pad, C]
// in tile order -> y [B, H, N_pad, D] (pad rows hold act(0)).
vsa_status launch_project(const vsa_plan_s* p, const void* x, const void* w, int B, int H, int D,
                          int C, int act, int tiled, void* y, cudaStream_t stream);

// Backward (backward.cu).
size_t colmask_bytes(const vsa_plan_s* p, int64_t bh);
size_t coarse_bwd_bytes(const vsa_plan_s* p, int64_t bh);
cudaError_t launch_combine_backward(const vsa_plan_s* p, const void* d_out_t, const void* o_fine_t,
                                    const void* gate_t, const float* o_coarse, int64_t bh, int D,
                                    float* delta, void* d_gate_t, float* d_oc, cudaStream_t stream);
cudaError_t launch_coarse_backward(const vsa_plan_s* p, const float* qbar, const float* kbar,
                                   const float* vbar, const float* d_oc, int64_t bh, int D,
                                   float scale, float* d_qbar, float* d_kbar, float* d_vbar,
                                   void* ws, cudaStream_t stream);
// k_ref < 0: every reference tile (topk_ref ignored).
vsa_status launch_sparse_attn_backward(const vsa_plan_s* p, const void* q_t, const void* k_t,
                                       const void* v_t, const void* d_out_t,
                                       const int32_t* topk_idx, int k, const int32_t* topk_ref,
                                       int k_ref, const float* lse_t, const float* delta,
                                       const float* d_qbar, const float* d_kbar,
                                       const float* d_vbar, int64_t bh, int D, float scale,
                                       void* dq_t, void* dk_t, void* dv_t, void* ws,
                                       cudaStream_t stream);

// Self-test of the bounded wait (selftest.cu): result int32[2], 0 = the wait gave up.
cudaError_t launch_bounded_wait_check(unsigned int* status, int* result, cudaStream_t stream);

// Device status codes written by kernels into vsa_plan_s::d_status.
enum : unsigned int { kStatusOk = 0, kStatusTimeout = 1, kStatusBadIndex = 2 };

}  // namespace vsa
