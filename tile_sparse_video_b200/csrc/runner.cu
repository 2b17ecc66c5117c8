// vsa_runner: the whole layer over inputs in host memory, with the transfers
// overlapped with the computation.
//
// Three streams and two sets of device buffers: while layer i computes on
// the compute stream, the inputs of layer i+1 are copied in on the copy-in
// stream and the output of layer i-1 is copied out on the copy-out stream.
// Per buffer set, events order the reuse: a set's inputs are overwritten only
// after the layer that read them has finished, and its output only after it
// was copied out.  Each layer is the fused five-launch chain (permute + pool of
// Q, K and V, coarse attention + top-k from the pooled means, block-sparse
// attention with the gated combine in its epilogue, natural order).  Host
// buffers should be pinned (page-locked) for the copies to be asynchronous.
#include <cuda_runtime.h>

#include <new>
#include <string>

#include "vsa_internal.h"

struct vsa_runner_s {
  vsa_plan_s* plan = nullptr;
  int B = 0, H = 0, D = 0, k = 0;
  float scale = 0.f;
  size_t in_bytes = 0, tiled_bytes = 0, ws_bytes = 0;
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  cudaEvent_t t_start = nullptr, t_end = nullptr;   // timing of the last run
  bool timed = false;
  struct Set {
    void* in[4] = {};             // natural q, k, v, g [B,H,N,D] bf16
    void* tiled[3] = {};          // permuted q, k, v [B,H,N_pad,D] bf16
    void* ws = nullptr;           // pooled means + coarse score rows
    float* o_coarse = nullptr;    // [B,H,T,D] fp32
    int32_t* topk = nullptr;      // [B,H,n_v,k]
    void* out = nullptr;          // [B,H,N,D] bf16
    cudaEvent_t in_done = nullptr, comp_done = nullptr, out_done = nullptr;
  } set[2];
};

namespace {

vsa_status runner_cuda(cudaError_t e, const char* what) {
  return vsa::fail(VSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

void runner_free(vsa_runner_s* r) {
  for (auto& s : r->set) {
    for (void* p : s.in) cudaFree(p);
    for (void* p : s.tiled) cudaFree(p);
    cudaFree(s.ws);
    cudaFree(s.o_coarse);
    cudaFree(s.topk);
    cudaFree(s.out);
    if (s.in_done) cudaEventDestroy(s.in_done);
    if (s.comp_done) cudaEventDestroy(s.comp_done);
    if (s.out_done) cudaEventDestroy(s.out_done);
  }
  for (cudaStream_t st : {r->s_in, r->s_comp, r->s_out})
    if (st) cudaStreamDestroy(st);
  if (r->t_start) cudaEventDestroy(r->t_start);
  if (r->t_end) cudaEventDestroy(r->t_end);
  delete r;
}

}  // namespace

extern "C" {

vsa_status vsa_runner_create(vsa_plan p, int B, int H, int D, int k, float scale, vsa_runner* out) {
  if (p == nullptr || out == nullptr) return vsa::fail(VSA_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  if (p->device < 0) return vsa::fail(VSA_ERR_INVALID_ARG, "host-only plan (device = -1)");
  if (B <= 0 || H <= 0) return vsa::fail(VSA_ERR_INVALID_ARG, "B and H must be > 0");
  if (D != 64 && D != 128) return vsa::fail(VSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128");
  const int n_v = p->n_tiles - p->n_prefix_tiles;
  if (k < 0 || k > n_v) return vsa::fail(VSA_ERR_INVALID_ARG, "k outside [0, n_v]");
  if (k == 0 && p->n_prefix_tiles == 0)
    return vsa::fail(VSA_ERR_INVALID_ARG, "k = 0 with no prefix tile leaves a query without keys");
  if (!(scale > 0.0f)) return vsa::fail(VSA_ERR_INVALID_ARG, "scale must be > 0");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return runner_cuda(e, "cudaGetDevice");
  if (cur != p->device)
    return vsa::fail(VSA_ERR_INVALID_ARG, "current CUDA device differs from the plan's device");
  vsa_runner_s* r = new (std::nothrow) vsa_runner_s();
  if (r == nullptr) return vsa::fail(VSA_ERR_INVALID_ARG, "out of host memory");
  r->plan = p;
  r->B = B;
  r->H = H;
  r->D = D;
  r->k = k;
  r->scale = scale;
  const size_t bhd = size_t(B) * H * D;
  r->in_bytes = bhd * p->n_tokens * 2;
  r->tiled_bytes = bhd * p->n_padded * 2;
  size_t ws = 0;
  vsa_status st = vsa_workspace_size(p, B, H, D, k, &ws);
  if (st != VSA_OK) {
    delete r;
    return st;
  }
  r->ws_bytes = ws;
  for (auto& s : r->set) {
    for (void*& q : s.in)
      if (e == cudaSuccess) e = cudaMalloc(&q, r->in_bytes);
    for (void*& q : s.tiled)
      if (e == cudaSuccess) e = cudaMalloc(&q, r->tiled_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&s.ws, ws);
    if (e == cudaSuccess) e = cudaMalloc(&s.o_coarse, bhd * p->n_tiles * 4);
    if (e == cudaSuccess) e = cudaMalloc(&s.topk, size_t(B) * H * n_v * (k > 0 ? k : 1) * 4);
    if (e == cudaSuccess) e = cudaMalloc(&s.out, r->in_bytes);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.in_done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.comp_done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.out_done, cudaEventDisableTiming);
  }
  for (cudaStream_t* st2 : {&r->s_in, &r->s_comp, &r->s_out})
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(st2, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreate(&r->t_start);
  if (e == cudaSuccess) e = cudaEventCreate(&r->t_end);
  if (e != cudaSuccess) {
    runner_free(r);
    return runner_cuda(e, "vsa_runner_create allocations");
  }
  *out = r;
  return VSA_OK;
}

vsa_status vsa_runner_run(vsa_runner r, int n_layers, const void* const* q, const void* const* k_in,
                          const void* const* v, const void* const* g, void* const* out,
                          void* stream) {
  VSA_NVTX_RANGE();
  if (r == nullptr) return vsa::fail(VSA_ERR_INVALID_ARG, "runner is NULL");
  if (n_layers < 0) return vsa::fail(VSA_ERR_INVALID_ARG, "n_layers < 0");
  if (n_layers == 0) return VSA_OK;
  if (q == nullptr || k_in == nullptr || v == nullptr || g == nullptr || out == nullptr)
    return vsa::fail(VSA_ERR_INVALID_ARG, "NULL pointer array");
  for (int i = 0; i < n_layers; ++i)
    if (q[i] == nullptr || k_in[i] == nullptr || v[i] == nullptr || g[i] == nullptr ||
        out[i] == nullptr)
      return vsa::fail(VSA_ERR_INVALID_ARG, "NULL host buffer for layer " + std::to_string(i));
  vsa_plan_s* p = r->plan;
  const cudaStream_t caller = static_cast<cudaStream_t>(stream);
  // the runner's streams start after everything already queued on the caller's
  cudaEvent_t go = nullptr;
  cudaError_t e = cudaEventCreateWithFlags(&go, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(go, caller);
  for (cudaStream_t st : {r->s_in, r->s_comp, r->s_out})
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, go, 0);
  if (e == cudaSuccess) e = cudaEventRecord(r->t_start, r->s_in);
  if (e != cudaSuccess) {
    if (go) cudaEventDestroy(go);
    return runner_cuda(e, "vsa_runner_run setup");
  }
  const void* const* host_in[4] = {q, k_in, v, g};
  vsa_status st = VSA_OK;
  for (int i = 0; i < n_layers && st == VSA_OK && e == cudaSuccess; ++i) {
    auto& s = r->set[i & 1];
    // copy-in: the set's inputs were last read by layer i-2
    if (i >= 2) e = cudaStreamWaitEvent(r->s_in, s.comp_done, 0);
    for (int x = 0; x < 4 && e == cudaSuccess; ++x)
      e = cudaMemcpyAsync(s.in[x], host_in[x][i], r->in_bytes, cudaMemcpyHostToDevice, r->s_in);
    if (e == cudaSuccess) e = cudaEventRecord(s.in_done, r->s_in);
    // compute: after the copy-in, and after layer i-2's output left the set
    if (e == cudaSuccess) e = cudaStreamWaitEvent(r->s_comp, s.in_done, 0);
    if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(r->s_comp, s.out_done, 0);
    if (e != cudaSuccess) break;
    const size_t n_means = size_t(r->B) * r->H * p->n_tiles * r->D;
    float* pooled = static_cast<float*>(s.ws);
    for (int x = 0; x < 3 && st == VSA_OK; ++x)
      st = vsa_permute_pool(p, s.in[x], s.tiled[x], r->B, r->H, r->D, pooled + x * n_means,
                            r->s_comp);
    if (st == VSA_OK)
      st = vsa_coarse_topk_pooled(p, r->B, r->H, r->D, r->scale, r->k, s.o_coarse, s.topk, nullptr,
                                  s.ws, r->ws_bytes, r->s_comp);
    if (st == VSA_OK)
      st = vsa_sparse_attn_combine(p, s.tiled[0], s.tiled[1], s.tiled[2], s.topk, r->B, r->H,
                                   r->D, r->k, r->scale, s.in[3], s.o_coarse, s.out, nullptr,
                                   r->s_comp);
    if (st != VSA_OK) break;
    e = cudaEventRecord(s.comp_done, r->s_comp);
    // copy-out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(r->s_out, s.comp_done, 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(out[i], s.out, r->in_bytes, cudaMemcpyDeviceToHost, r->s_out);
    if (e == cudaSuccess) e = cudaEventRecord(s.out_done, r->s_out);
  }
  if (e == cudaSuccess && st == VSA_OK) e = cudaEventRecord(r->t_end, r->s_out);
  // the caller's stream continues after the last copy-out
  if (e == cudaSuccess && st == VSA_OK) e = cudaStreamWaitEvent(caller, r->t_end, 0);
  cudaEventDestroy(go);
  if (st != VSA_OK) return st;
  if (e != cudaSuccess) return runner_cuda(e, "vsa_runner_run");
  r->timed = true;
  return VSA_OK;
}

vsa_status vsa_runner_elapsed(vsa_runner r, float* ms) {
  if (r == nullptr || ms == nullptr) return vsa::fail(VSA_ERR_INVALID_ARG, "NULL argument");
  if (!r->timed) return vsa::fail(VSA_ERR_INVALID_ARG, "no run to time");
  cudaError_t e = cudaEventSynchronize(r->t_end);
  if (e == cudaSuccess) e = cudaEventElapsedTime(ms, r->t_start, r->t_end);
  return e == cudaSuccess ? VSA_OK : runner_cuda(e, "vsa_runner_elapsed");
}

vsa_status vsa_runner_destroy(vsa_runner r) {
  if (r == nullptr) return VSA_OK;
  cudaStreamSynchronize(r->s_in);
  cudaStreamSynchronize(r->s_comp);
  cudaStreamSynchronize(r->s_out);
  runner_free(r);
  return VSA_OK;
}

}  // extern "C"
