// Backward pass of the tile-sparse attention layer, for sm_100a.
//
// The layer is trained end to end (SnackOnAI, "The Architecture, Unpacked":
// the coarse stage and the gate are learned; the VSA paper it builds on trains
// its sparse kernel).  The top-k selection is an index choice and passes no
// gradient; everything else is differentiated from its definition:
//
//   combine   out = o_fine + sigmoid(g) * o_coarse[tile]          (live rows)
//             -> d_g = d_out * o_coarse[tile] * s (1 - s),  s = sigmoid(g)
//                d_o_coarse[t] = sum over the live rows of t of d_out * s
//                delta[r] = <d_out[r], o_fine[r]>  (the row statistic of the
//                           softmax backward below)
//   coarse    s = scale qbar kbar^T, P = softmax_rows(s), o_coarse = P vbar
//             -> d_vbar = P^T d_oc, dS = P * (d_oc vbar^T - rowsum(P * d_oc vbar^T)),
//                d_qbar = scale dS kbar, d_kbar = scale dS^T qbar
//   fine      for each query tile i and key tile j of its key set:
//             P = exp(scale Q_i K_j^T - lse_i), dP = dO_i V_j^T,
//             dS = P * (dP - delta_i); dQ_i += scale dS K_j,
//             dK_j += scale dS^T Q_i, dV_j += P^T dO_i
//   pool      each live row of tile t receives d_bar[t] / block_len[t]
//
// Kernels:
//   combine_bwd_kernel   one warp per (b*h, tile): HBM-bound, one pass over
//                        d_out, o_fine and g.
//   sgemm_kernel + softmax row kernels: the coarse backward on the pooled
//                        [T, D] matrices (small, fp32 on the CUDA cores).
//   colmask_kernel       for every key tile, the bitmap of the query tiles
//                        that attend to it (the transpose of the selection).
//   attn_bwd_kernel<R, D, kKeyMajor>: tcgen05 kernel, one persistent CTA per
//                        SM taking work items from a global counter.
//                        Query-major (dQ): item = (b*h, query tile i), loop
//                        over its key tiles.  Key-major (dK, dV): item = (b*h,
//                        key tile j), loop over the query tiles whose key set
//                        holds j.  Each step is split into 64-column
//                        half-steps that alternate between two elementwise
//                        warpgroups and two TMEM buffers: the score-side
//                        products go to TMEM (S and dP, M=128, N=64, K=D), the
//                        warpgroup turns them into bf16 P / dS in TMEM, and
//                        TS-MMAs accumulate dQ (or dK and dV) in TMEM.  The
//                        epilogue adds the pooling term and writes bf16.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <string>

#include "vsa_internal.h"
#include "sm100.cuh"

namespace vsa {
namespace {

using namespace sm100;

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint16_t h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// ---------------------------------------------------------------- combine backward

// One warp per (b*h, tile t); lane owns D/32 consecutive columns.  Rows past
// block_len[t] get d_g = 0 and delta = 0.
template <int D>
__global__ void __launch_bounds__(256) combine_bwd_kernel(
    const uint16_t* __restrict__ d_out, const uint16_t* __restrict__ o_fine,
    const uint16_t* __restrict__ gate, const float* __restrict__ o_coarse,
    const int32_t* __restrict__ block_len, float* __restrict__ delta, uint16_t* __restrict__ d_gate,
    float* __restrict__ d_oc, int64_t n_items, int T, int R) {
  constexpr int E = D / 32;
  const int64_t item = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= n_items) return;
  const int lane = threadIdx.x & 31;
  const int64_t bh = item / T;
  const int t = int(item % T);
  const int blen = __ldg(block_len + t);
  const int64_t row0 = (bh * T + t) * int64_t(R);
  float oc[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    oc[e] = __ldg(o_coarse + (bh * T + t) * D + lane * E + e);
    acc[e] = 0.f;
  }
#pragma unroll 4
  for (int r = 0; r < R; ++r) {
    const int64_t off = (row0 + r) * D + lane * E;
    uint16_t dv[E], ov[E], gv[E];
    if (r < blen) {
      if (E == 4) {
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(d_out + off));
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(o_fine + off));
        const uint2 c = __ldg(reinterpret_cast<const uint2*>(gate + off));
        const uint32_t aa[2] = {a.x, a.y}, bb[2] = {b.x, b.y}, cc[2] = {c.x, c.y};
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dv[e] = uint16_t(aa[e / 2] >> (16 * (e & 1)));
          ov[e] = uint16_t(bb[e / 2] >> (16 * (e & 1)));
          gv[e] = uint16_t(cc[e / 2] >> (16 * (e & 1)));
        }
      } else {
        const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(d_out + off));
        const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(o_fine + off));
        const uint32_t c = __ldg(reinterpret_cast<const uint32_t*>(gate + off));
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dv[e] = uint16_t(a >> (16 * e));
          ov[e] = uint16_t(b >> (16 * e));
          gv[e] = uint16_t(c >> (16 * e));
        }
      }
      float dot = 0.f;
      uint16_t dg[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float d = bf16_to_f32(dv[e]);
        const float s = 1.f / (1.f + __expf(-bf16_to_f32(gv[e])));
        dot = fmaf(d, bf16_to_f32(ov[e]), dot);
        acc[e] = fmaf(d, s, acc[e]);
        dg[e] = f32_to_bf16(d * oc[e] * s * (1.f - s));
      }
      dot = warp_sum(dot);
      if (lane == 0) delta[row0 + r] = dot;
      if (E == 4) {
        *reinterpret_cast<uint2*>(d_gate + off) =
            make_uint2(uint32_t(dg[0]) | (uint32_t(dg[1]) << 16), uint32_t(dg[2]) | (uint32_t(dg[3]) << 16));
      } else {
        *reinterpret_cast<uint32_t*>(d_gate + off) = uint32_t(dg[0]) | (uint32_t(dg[1]) << 16);
      }
    } else {
      if (lane == 0) delta[row0 + r] = 0.f;
      if (E == 4)
        *reinterpret_cast<uint2*>(d_gate + off) = make_uint2(0u, 0u);
      else
        *reinterpret_cast<uint32_t*>(d_gate + off) = 0u;
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) d_oc[(bh * T + t) * D + lane * E + e] = acc[e];
}

// ---------------------------------------------------------------- coarse backward

// Batched fp32 GEMM on the CUDA cores: C[b] (M x N, row-major) =
// alpha * sum_k A(b, m, k) B(b, k, n), with A(b, m, k) = A[b*sab + m*sam + k*sak]
// and B(b, k, n) = B[b*sbb + k*sbk + n*sbn].  64 x 64 tiles, 256 threads,
// 4 x 4 outputs per thread.
constexpr int kGB = 64, kGK = 16;

__global__ void __launch_bounds__(256) sgemm_kernel(const float* __restrict__ A,
                                                    const float* __restrict__ B, float* __restrict__ C,
                                                    int M, int N, int K, int64_t sab, int64_t sam,
                                                    int64_t sak, int64_t sbb, int64_t sbk,
                                                    int64_t sbn, float alpha) {
  __shared__ float As[kGK][kGB + 4];
  __shared__ float Bs[kGK][kGB + 4];
  const int64_t b = blockIdx.z;
  const int m0 = blockIdx.y * kGB, n0 = blockIdx.x * kGB;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const float* Ab = A + b * sab;
  const float* Bb = B + b * sbb;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kGK) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = tid + 256 * u;
      // walk the contiguous dimension with consecutive threads
      int m, k;
      if (sak == 1) { m = e / kGK; k = e % kGK; } else { m = e % kGB; k = e / kGB; }
      As[k][m] = (m0 + m < M && k0 + k < K) ? __ldg(Ab + (m0 + m) * sam + (k0 + k) * sak) : 0.f;
      int n, kb;
      if (sbn == 1) { n = e % kGB; kb = e / kGB; } else { n = e / kGK; kb = e % kGK; }
      Bs[kb][n] = (n0 + n < N && k0 + kb < K) ? __ldg(Bb + (k0 + kb) * sbk + (n0 + n) * sbn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* Cb = C + b * int64_t(M) * N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) Cb[int64_t(m) * N + n] = alpha * acc[i][j];
    }
  }
}

// Row-wise softmax in place: one warp per row of length T.
__global__ void __launch_bounds__(256) softmax_rows_kernel(float* __restrict__ s, int64_t rows, int T) {
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float* x = s + row * T;
  float m = -INFINITY;
  for (int j = lane; j < T; j += 32) m = fmaxf(m, x[j]);
  m = warp_max(m);
  float l = 0.f;
  for (int j = lane; j < T; j += 32) l += __expf(x[j] - m);
  l = warp_sum(l);
  const float inv = 1.f / l;
  for (int j = lane; j < T; j += 32) x[j] = __expf(x[j] - m) * inv;
}

// dS = P * (dP - rowsum(P * dP)) in place over dP: one warp per row.
__global__ void __launch_bounds__(256) softmax_bwd_rows_kernel(const float* __restrict__ p,
                                                               float* __restrict__ dp, int64_t rows,
                                                               int T) {
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const float* pr = p + row * T;
  float* dr = dp + row * T;
  float s = 0.f;
  for (int j = lane; j < T; j += 32) s = fmaf(pr[j], dr[j], s);
  s = warp_sum(s);
  for (int j = lane; j < T; j += 32) dr[j] = pr[j] * (dr[j] - s);
}

// ---------------------------------------------------------------- selection transpose

// Bit i of word (bh, j, i / 32) is set when query tile i attends to key tile
// j: every j for a prefix query tile, else its reference tiles (all n_p, or
// its k_ref listed ones) and its k kept video tiles.  One warp per (bh, i);
// the bitmap must be zero on entry.  An index outside its range is skipped
// and recorded.
__global__ void __launch_bounds__(256) colmask_kernel(
    const int32_t* __restrict__ topk, const int32_t* __restrict__ topk_ref, uint32_t* colmask,
    unsigned int* status, int64_t n_items, int T, int n_p, int k, int k_ref, int n_sink, int W) {
  const int64_t item = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= n_items) return;
  const int lane = threadIdx.x & 31;
  const int64_t bh = item / T;
  const int i = int(item % T);
  const uint32_t bit = 1u << (i & 31);
  uint32_t* base = colmask + bh * int64_t(T) * W + (i >> 5);
  if (i < n_p) {
    for (int j = lane; j < T; j += 32) atomicOr(base + int64_t(j) * W, bit);
    return;
  }
  const int n_v = T - n_p;
  const int64_t rowi = bh * n_v + (i - n_p);
  for (int x = lane; x < n_sink + k; x += 32) {
    int j;
    if (x < n_sink) {
      j = topk_ref != nullptr ? __ldg(topk_ref + rowi * k_ref + x) : x;
      if (j < 0 || j >= n_p) { record(status, kStatusBadIndex, unsigned(j)); continue; }
    } else {
      j = __ldg(topk + rowi * k + (x - n_sink));
      if (j < n_p || j >= T) { record(status, kStatusBadIndex, unsigned(j)); continue; }
    }
    atomicOr(base + int64_t(j) * W, bit);
  }
}

// ---------------------------------------------------------------- fine backward (tcgen05)

constexpr int kThreadsBwd = 320;   // warps 0-7 elementwise + epilogue, 8 lists/TMA/S-dP MMA, 9 accumulating MMA
constexpr int kBwdM = 128;         // MMA rows: one row tile (rows at or past R are ignored)
constexpr int kWarpIssue = 8;
constexpr int kWarpAcc = 9;

struct BwdArgs {
  const int32_t* block_len;   // [T]
  const int32_t* topk;        // [BH, n_v, k]
  const int32_t* topk_ref;    // [BH, n_v, k_ref] or null (every reference tile)
  const uint32_t* colmask;    // key-major: [BH, T, W] query tiles of each key tile
  const float* lse;           // [BH, N_pad] natural-log row log-sum-exp (forward)
  const float* delta;         // [BH, N_pad] <d_out, o_fine> per row
  const float* dbar;          // [BH, T, D] pooled gradient of the first output, or null
  const float* dbar2;         // key-major: pooled gradient of dV, or null
  uint16_t* out;              // dQ_t (query-major) or dK_t (key-major), bf16 [BH, N_pad, D]
  uint16_t* out2;             // key-major: dV_t
  unsigned int* status;
  unsigned long long wait_ns; // bound of every mbarrier wait
  unsigned int* next_item;    // work counter (zero at launch)
  int T, n_p, k, k_ref, n_sink, W, n_items;
  int64_t n_pad;
  float scale, scale_log2;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Untiled bulk copy global -> shared, completing on an mbarrier (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Bounded wait taken by a whole warp: every lane waits, and the warp goes on
// only if all of them saw the phase (so that no lane is left behind at the
// warp-collective tcgen05 instructions that follow when the CTA aborts).
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* status, unsigned int where,
                                          unsigned long long limit_ns) {
  const bool ok = wait_bar(bar, parity, abort_flag, status, where, limit_ns);
  return __all_sync(0xFFFFFFFFu, ok);
}

// P and dS of 32 score columns of one row: P = 2^(S scale log2(e) - lse
// log2(e)) (0 at or past column `lim`), dS = P (dP - delta), as bf16 pairs.
// Query-major: lse and delta are the row's (nl2_row = -lse log2(e));
// key-major: the columns' (c_lse, c_del: 32 floats each in shared memory).
template <bool kKeyMajor, bool kMask>
__device__ __forceinline__ void p_and_ds_cols(const uint32_t (&sr)[32], const uint32_t (&dr)[32],
                                              float scale_log2, float nl2_row, float delta_row,
                                              const float* c_lse, const float* c_del, int lim,
                                              uint32_t (&pp)[16], uint32_t (&dd)[16]) {
  constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
    float nl[4], dl[4];
    if (kKeyMajor) {
      const float4 l4 = *reinterpret_cast<const float4*>(c_lse + 4 * q4);
      const float4 d4 = *reinterpret_cast<const float4*>(c_del + 4 * q4);
      nl[0] = -l4.x * kLog2e; nl[1] = -l4.y * kLog2e; nl[2] = -l4.z * kLog2e; nl[3] = -l4.w * kLog2e;
      dl[0] = d4.x; dl[1] = d4.y; dl[2] = d4.z; dl[3] = d4.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        nl[e] = nl2_row;
        dl[e] = delta_row;
      }
    }
    float pv[4], dv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = 4 * q4 + e;
      float p = ex2f(fmaf(__uint_as_float(sr[col]), scale_log2, nl[e]));
      if (kMask && col >= lim) p = 0.f;
      pv[e] = p;
      dv[e] = p * (__uint_as_float(dr[col]) - dl[e]);
    }
    pp[2 * q4] = pack_bf16(pv[0], pv[1]);
    pp[2 * q4 + 1] = pack_bf16(pv[2], pv[3]);
    dd[2 * q4] = pack_bf16(dv[0], dv[1]);
    dd[2 * q4 + 1] = pack_bf16(dv[2], dv[3]);
  }
}

template <bool kKeyMajor>
__device__ __forceinline__ void p_and_ds(const uint32_t (&sr)[32], const uint32_t (&dr)[32],
                                         float scale_log2, float nl2_row, float delta_row,
                                         const float* c_lse, const float* c_del, int lim,
                                         uint32_t (&pp)[16], uint32_t (&dd)[16]) {
  if (lim >= 32)   // every column live (the common case): no mask
    p_and_ds_cols<kKeyMajor, false>(sr, dr, scale_log2, nl2_row, delta_row, c_lse, c_del, lim, pp, dd);
  else
    p_and_ds_cols<kKeyMajor, true>(sr, dr, scale_log2, nl2_row, delta_row, c_lse, c_del, lim, pp, dd);
}

template <int R, int D, bool kKeyMajor>
struct BwdCfg {
  static constexpr int N = R;                       // rows of a column-side tile
  static constexpr int NH = 64;                     // score columns of a half-step
  static constexpr int HS = N / NH;                 // half-steps per step
  static constexpr int NS = HS == 1 ? 3 : 2;        // column-side ring stages
  static constexpr int XBYTES = kBwdM * D * 2;      // one row-side tile (128-row box)
  static constexpr int YBYTES = N * D * 2;          // one column-side tile
  static constexpr int CBYTES = 2 * N * 4;          // key-major: lse and delta of the column tile
  static constexpr int OFF_X1 = 0;
  static constexpr int OFF_X2 = XBYTES;
  static constexpr int OFF_Y = 2 * XBYTES;          // stage s: Y1 at + s*2*YBYTES, Y2 at + YBYTES
  static constexpr int OFF_C = OFF_Y + NS * 2 * YBYTES;   // stage s: + s*CBYTES
  static constexpr int OFF_BAR = OFF_C + NS * CBYTES;
  // barriers: x_full, y_full[NS], s_full[2], p_ready[2], acc_done[2], acc_full,
  //           list_full, epi_done, drain, drain2
  static constexpr int NBAR = 1 + NS + 6 + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;   // tmem slot, abort flag, list count
  static constexpr int OFF_LIST = OFF_MISC + 16;
  // TMEM columns: accumulators (dQ; or dK then dV), then two half-step
  // buffers, each S [NH columns] then dP [NH columns]
  static constexpr uint32_t COL_ACC0 = 0;
  static constexpr uint32_t COL_ACC1 = D;
  static constexpr uint32_t COL_BUF = kKeyMajor ? 2 * D : D;
  static constexpr uint32_t TMEM_COLS = (COL_BUF + 4 * NH) <= 256 ? 256u : 512u;
  static_assert(COL_BUF + 4 * NH <= 512, "TMEM columns");
  static_assert(N % NH == 0, "tile rows");
  static constexpr uint32_t IDESC_SS = idesc_bf16(kBwdM, NH, false, false);
  static constexpr uint32_t IDESC_ACC = idesc_bf16(kBwdM, D, false, true);
  // the list: column tile of each step int32[T], then its block_len int32[T]
  static size_t bytes(int T) { return size_t(OFF_LIST) + size_t(8) * ((T + 3) & ~3); }
};

// Work items are (b*h, row tile) in head-major order (each head's prefix
// tiles, then its video tiles), handed out in that order from a global
// counter.  The items' lengths vary (a key tile is attended by as many query
// tiles as selected it), and under a static round-robin split the CTAs drifted
// apart by several heads, whose column-side tiles then no longer shared the
// L2 (measured: 20x the algorithmic DRAM reads of the key-major kernel).
// Taken in order, the concurrent items stay within one or two heads.
__device__ __forceinline__ void decode_bwd_item(int item, int T, int64_t& bh, int& t) {
  bh = item / T;
  t = item % T;
}

// Half-step u of an item covers score columns [c*NH, (c+1)*NH) (c = u % HS)
// of step n = u / HS.  Half-steps alternate between the two elementwise
// warpgroups and their two TMEM buffers (w = global half-step & 1), so that
// one warpgroup's exponentials overlap the tensor core's work on the other's.
template <int R, int D, bool kKeyMajor>
__global__ void __launch_bounds__(kThreadsBwd, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ CUtensorMap tm_x2,
                    const __grid_constant__ CUtensorMap tm_y1, const __grid_constant__ CUtensorMap tm_y2,
                    const BwdArgs a) {
  using C = BwdCfg<R, D, kKeyMajor>;
  constexpr int N = C::N, NH = C::NH, HS = C::HS, NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sX1 = s_base + C::OFF_X1, sX2 = s_base + C::OFF_X2, sY = s_base + C::OFF_Y;
  const uint32_t bar0 = s_base + C::OFF_BAR;
  // x_full: row-side tiles of an item.  y_full[s]: column-side tiles (and, key-
  // major, their lse / delta) of the steps using stage s.  s_full[w],
  // p_ready[w] and acc_done[w] complete once per half-step of buffer w;
  // acc_full once per item with steps; list_full and epi_done once per item
  // (epi_done: the eight elementwise warps after the epilogue and the
  // accumulating warp after its last product of the item).
  // The issuer reuses buffer w (and reloads a stage) only after acc_done of
  // its previous half-step, which follows that half-step's p_ready, so no
  // waiter can fall two phases behind.
  const uint32_t x_full = bar0, y_full = bar0 + 8, s_full = y_full + 8 * NS, p_ready = s_full + 16,
                 acc_done = p_ready + 16, acc_full = acc_done + 16, list_full = acc_full + 8,
                 epi_done = list_full + 8, drain = epi_done + 8, drain2 = drain + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* s_cnt = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  volatile int* s_item = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 12);
  int32_t* s_list = reinterpret_cast<int32_t*>(smem + C::OFF_LIST);
  int32_t* s_blen = s_list + ((a.T + 3) & ~3);
  const float* s_c = reinterpret_cast<const float*>(smem + C::OFF_C);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(x_full, 1);
    for (int s = 0; s < NS; ++s) mbar_init(y_full + 8 * s, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(s_full + 8 * w, 1);
      mbar_init(p_ready + 8 * w, 4);
      mbar_init(acc_done + 8 * w, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(list_full, 1);
    mbar_init(epi_done, 9);          // 8 elementwise warps + the accumulating warp
    mbar_init(drain, 1);
    mbar_init(drain2, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpIssue) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_x1);
      tma_prefetch_desc(&tm_x2);
      tma_prefetch_desc(&tm_y1);
      tma_prefetch_desc(&tm_y2);
    }
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpIssue) {
    // ------------------------------------------------------------ lists, TMA, MMA
    uint32_t G = 0, Gs = 0;           // half-steps / steps of earlier items
    uint32_t hw[2] = {0, 0};          // half-steps of each buffer so far
    uint32_t x_loads = 0;
    uint32_t y_issued[NS] = {}, y_seen[NS] = {};
    bool x_pending = false;
    int t = 0;
    bool ok = true;
    for (; ok; ++t) {
      // the previous item's epilogue is done with the accumulators and the list
      if (t > 0 && !wait_warp(epi_done, (t - 1) & 1, abort_flag, a.status, 40, a.wait_ns)) { ok = false; break; }
      int item = 0;
      if (lane == 0) item = int(atomicAdd(a.next_item, 1u));
      item = __shfl_sync(0xFFFFFFFFu, item, 0);
      if (item >= a.n_items) {
        if (lane == 0) {
          *s_item = -1;               // tells the elementwise warps to stop
          mbar_arrive(list_full);
        }
        break;
      }
      int64_t bh;
      int rt;
      decode_bwd_item(item, a.T, bh, rt);
      int cnt = 0;
      if (kKeyMajor) {
        // query tiles whose key set holds key tile rt, ascending
        const uint32_t* row = a.colmask + (bh * a.T + rt) * int64_t(a.W);
        for (int base = 0; base < a.W; base += 32) {
          const int wd = base + lane;
          uint32_t word = wd < a.W ? __ldg(row + wd) : 0u;
          const int c = __popc(word);
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
          }
          int pos = cnt + incl - c;
          while (word != 0u) {
            s_list[pos++] = 32 * wd + (__ffs(word) - 1);
            word &= word - 1u;
          }
          cnt += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
      } else if (rt < a.n_p) {
        cnt = a.T;                    // prefix query tiles attend densely
        for (int x = lane; x < cnt; x += 32) s_list[x] = x;
      } else {
        cnt = a.n_sink + a.k;
        const int64_t rowi = bh * (a.T - a.n_p) + (rt - a.n_p);
        for (int x = lane; x < cnt; x += 32) {
          int j;
          if (x < a.n_sink) {
            j = a.topk_ref != nullptr ? __ldg(a.topk_ref + rowi * a.k_ref + x) : x;
            if (j < 0 || j >= a.n_p) { record(a.status, kStatusBadIndex, unsigned(j)); j = 0; }
          } else {
            j = __ldg(a.topk + rowi * a.k + (x - a.n_sink));
            if (j < a.n_p || j >= a.T) { record(a.status, kStatusBadIndex, unsigned(j)); j = a.n_p; }
          }
          s_list[x] = j;
        }
      }
      __syncwarp();
      for (int x = lane; x < cnt; x += 32) s_blen[x] = __ldg(a.block_len + s_list[x]);
      __threadfence_block();
      __syncwarp();
      if (lane == 0) {
        *s_cnt = cnt;
        *s_item = item;
        mbar_arrive(list_full);
        const int64_t row0 = bh * a.n_pad;
        const int U = cnt * HS;
        auto load_y = [&](int n) {
          const uint32_t s = (Gs + n) % NS;
          const int j = s_list[n];
          const int r = int(row0 + int64_t(j) * R);
          const uint32_t bar = y_full + 8 * s;
          mbar_expect_tx(bar, 2 * C::YBYTES + (kKeyMajor ? C::CBYTES : 0));
          const uint32_t d1 = sY + s * 2 * C::YBYTES, d2 = d1 + C::YBYTES;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(d1 + c * N * 128, &tm_y1, bar, c * 64, r);
            tma_load_2d(d2 + c * N * 128, &tm_y2, bar, c * 64, r);
          }
          if (kKeyMajor) {
            const uint32_t dc = s_base + C::OFF_C + s * C::CBYTES;
            bulk_load(dc, a.lse + row0 + int64_t(j) * R, N * 4, bar);
            bulk_load(dc + N * 4, a.delta + row0 + int64_t(j) * R, N * 4, bar);
          }
          ++y_issued[s];
        };
        // S (or S^T) and dP (or dP^T) of half-step u into buffer (G + u) & 1
        auto issue_sd = [&](int u) -> bool {
          const int n = u / HS, c = u % HS;
          const uint32_t s = (Gs + n) % NS, w = (G + u) & 1;
          if (u == 0) {
            if (!wait_bar(x_full, (x_loads - 1) & 1, abort_flag, a.status, 41, a.wait_ns)) return false;
            x_pending = false;
          }
          if (c == 0) {
            if (!wait_bar(y_full + 8 * s, ((Gs + n) / NS) & 1, abort_flag, a.status, 42, a.wait_ns)) return false;
            ++y_seen[s];
          }
          tc_fence_after();
          const uint32_t y1 = sY + s * 2 * C::YBYTES, y2 = y1 + C::YBYTES;
          const uint32_t buf = tmem + C::COL_BUF + w * 2 * NH;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t ko = (ks / 4) * 128u * 128u + (ks % 4) * 32u;
            const uint32_t kn = (ks / 4) * uint32_t(N) * 128u + uint32_t(c * NH) * 128u + (ks % 4) * 32u;
            umma_bf16(buf, sdesc_sw128(sX1 + ko, 16, 1024), sdesc_sw128(y1 + kn, 16, 1024), C::IDESC_SS,
                      ks > 0 ? 1u : 0u);
            umma_bf16(buf + NH, sdesc_sw128(sX2 + ko, 16, 1024), sdesc_sw128(y2 + kn, 16, 1024),
                      C::IDESC_SS, ks > 0 ? 1u : 0u);
          }
          umma_commit(s_full + 8 * w);
          return true;
        };
        if (cnt > 0) {
          mbar_expect_tx(x_full, 2 * C::XBYTES);
          const int r = int(row0 + int64_t(rt) * R);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d_hint(sX1 + c * kBwdM * 128, &tm_x1, x_full, c * 64, r, l2_evict_first_policy());
            tma_load_2d_hint(sX2 + c * kBwdM * 128, &tm_x2, x_full, c * 64, r, l2_evict_first_policy());
          }
          ++x_loads;
          x_pending = true;
          for (int n = 0; n < cnt && n < NS; ++n) load_y(n);
          ok = issue_sd(0) && (U < 2 || issue_sd(1));
        }
        for (int u = 0; u < U && ok; ++u) {
          const int n = u / HS, c = u % HS;
          const uint32_t w = (G + u) & 1;
          const uint32_t idx = hw[w]++;
          if (u + 2 < U) {
            // buffer w (and, after a step's last half, its stage) is free once
            // the accumulating products of half-step u (warp kWarpAcc) have read it
            if (!wait_bar(acc_done + 8 * w, idx & 1, abort_flag, a.status, 44, a.wait_ns)) { ok = false; break; }
            if (c == HS - 1 && n + NS < cnt) load_y(n + NS);
            if (!issue_sd(u + 2)) { ok = false; break; }
          }
        }
        G += U;
        Gs += cnt;
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      G = __shfl_sync(0xFFFFFFFFu, G, 0);
      Gs = __shfl_sync(0xFFFFFFFFu, Gs, 0);
      __syncwarp();
    }
    if (lane == 0 && !ok) {
      // Abort: let every MMA issued above complete and every TMA copy land.
      umma_commit(drain);
      wait_bar_drain(drain, 0);
      for (int s = 0; s < NS; ++s)
        if (y_issued[s] > y_seen[s]) wait_bar_drain(y_full + 8 * s, (y_issued[s] - 1) & 1);
      if (x_pending) wait_bar_drain(x_full, (x_loads - 1) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpAcc) {
    // ------------------------------------------------------------ accumulating MMAs
    // dQ += dS K_j (or dK += dS^T Q_i, dV += P^T dO_i) of each half-step once
    // its warpgroup has written P / dS; a warp of its own, so that one
    // buffer's accumulation never waits behind the other buffer's products.
    uint32_t G = 0, Gs = 0;
    uint32_t hw[2] = {0, 0};
    int t = 0;
    bool ok = true;
    for (; ok; ++t) {
      if (!wait_warp(list_full, t & 1, abort_flag, a.status, 50, a.wait_ns)) { ok = false; break; }
      const int item = *s_item;
      if (item < 0) break;
      const int cnt = *s_cnt;
      const int U = cnt * HS;
      if (lane == 0) {
        for (int u = 0; u < U; ++u) {
          const int n = u / HS, c = u % HS;
          const uint32_t s = (Gs + n) % NS, w = (G + u) & 1;
          const uint32_t idx = hw[w]++;
          if (!wait_bar(p_ready + 8 * w, idx & 1, abort_flag, a.status, 43, a.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t y1 = sY + s * 2 * C::YBYTES, y2 = y1 + C::YBYTES;
          const uint32_t buf = tmem + C::COL_BUF + w * 2 * NH;
#pragma unroll
          for (int ks = 0; ks < NH / 16; ++ks) {
            const uint32_t boff = uint32_t(c * NH + ks * 16) * 128u;
            const uint32_t acc = (u > 0 || ks > 0) ? 1u : 0u;
            if (kKeyMajor) {
              // dK += dS^T Q_i,  dV += P^T dO_i   (B operands MN-major; bf16 pairs in
              // the first NH/2 columns of the dP and S halves of the buffer)
              umma_bf16_ts(tmem + C::COL_ACC0, buf + NH + ks * 8,
                           sdesc_sw128(y1 + boff, N * 128, 1024), C::IDESC_ACC, acc);
              umma_bf16_ts(tmem + C::COL_ACC1, buf + ks * 8, sdesc_sw128(y2 + boff, N * 128, 1024),
                           C::IDESC_ACC, acc);
            } else {
              // dQ += dS K_j
              umma_bf16_ts(tmem + C::COL_ACC0, buf + ks * 8, sdesc_sw128(y1 + boff, N * 128, 1024),
                           C::IDESC_ACC, acc);
            }
          }
          umma_commit(acc_done + 8 * w);
          if (u == U - 1) umma_commit(acc_full);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      G += U;
      Gs += cnt;
      // this warp is done with the item's list: the next one may be published
      // (without this arrival an item with no steps could let the list barrier
      // run two phases ahead of this warp)
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(epi_done);
    }
    if (lane == 0 && !ok) {
      // Abort: let every MMA this warp issued complete.
      umma_commit(drain2);
      wait_bar_drain(drain2, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise + epilogue
    // Warpgroup wg (warps 4wg .. 4wg+3) takes the half-steps of buffer wg;
    // thread = row of the row tile = TMEM lane.  In the epilogue warpgroup wg
    // writes accumulator columns [wg D/2, (wg+1) D/2).
    constexpr float kLog2e = 1.4426950408889634f;
    const int quad = warp & 3, wg = warp >> 2;
    const int row = quad * 32 + lane;
    const bool rows_active = (R == 128) || (quad < 2);
    const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
    const uint32_t buf = t_lane + C::COL_BUF + wg * 2 * NH;
    uint32_t G = 0, Gs = 0, mine = 0, accs = 0;
    int t = 0;
    bool ok = true;
    for (; ok; ++t) {
      if (!wait_warp(list_full, t & 1, abort_flag, a.status, 45, a.wait_ns)) { ok = false; break; }
      const int item = *s_item;
      if (item < 0) break;
      int64_t bh;
      int rt;
      decode_bwd_item(item, a.T, bh, rt);
      const int cnt = *s_cnt;
      const int U = cnt * HS;
      const int blen_row = __ldg(a.block_len + rt);
      float nl2_row = 0.f, delta_row = 0.f;       // query-major: -lse*log2(e) and delta of the row
      if (!kKeyMajor && rows_active && row < blen_row) {
        const int64_t r = bh * a.n_pad + int64_t(rt) * R + row;
        nl2_row = -__ldg(a.lse + r) * kLog2e;
        delta_row = __ldg(a.delta + r);
      }
      for (int u = int((uint32_t(wg) - G) & 1u); u < U; u += 2) {
        const int n = u / HS, c = u % HS;
        const uint32_t s = (Gs + n) % NS;
        if (!wait_warp(s_full + 8 * wg, mine & 1, abort_flag, a.status, 46, a.wait_ns)) { ok = false; break; }
        ++mine;
        if (kKeyMajor && !wait_warp(y_full + 8 * s, ((Gs + n) / NS) & 1, abort_flag, a.status, 47, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int blen_col = s_blen[n];
        if (rows_active) {
          const float* c_lse = s_c + s * (C::CBYTES / 4) + c * NH;
          const float* c_del = c_lse + N;
          const int lim = blen_col - c * NH;           // live score columns of this half-step
#pragma unroll
          for (int cc = 0; cc < NH / 32; ++cc) {
            uint32_t sr[32], dr[32], pp[16], dd[16];
            tmem_ld32(buf + cc * 32, sr);
            tmem_ld32(buf + NH + cc * 32, dr);
            tmem_wait_ld(sr);
            tmem_wait_ld(dr);
            p_and_ds<kKeyMajor>(sr, dr, a.scale_log2, nl2_row, delta_row, c_lse + cc * 32,
                                c_del + cc * 32, lim - cc * 32, pp, dd);
            // bf16 pairs into columns this thread has already read
            if (kKeyMajor) {
              tmem_st16(buf + cc * 16, pp);
              tmem_st16(buf + NH + cc * 16, dd);
            } else {
              tmem_st16(buf + cc * 16, dd);
            }
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready + 8 * wg);
      }
      if (!ok) break;
      G += U;
      Gs += cnt;
      // epilogue: accumulator (x scale for dQ, dK) + pooled gradient / block_len
      if (cnt > 0) {
        if (!wait_warp(acc_full, accs & 1, abort_flag, a.status, 48, a.wait_ns)) { ok = false; break; }
        ++accs;
        tc_fence_after();
      }
      if (rows_active) {
        const bool live = row < blen_row;
        const int64_t orow = bh * a.n_pad + int64_t(rt) * R + row;
        const float inv_blen = 1.f / float(blen_row);
#pragma unroll
        for (int o = 0; o < (kKeyMajor ? 2 : 1); ++o) {
          uint16_t* dst = (o == 0 ? a.out : a.out2) + orow * D;
          const float* pb = o == 0 ? a.dbar : a.dbar2;
          const float mult = o == 0 ? a.scale : 1.f;
          const uint32_t col_acc = o == 0 ? C::COL_ACC0 : C::COL_ACC1;
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) {
            const int c0 = wg * (D / 2) + cc * 32;
            uint32_t v[32];
            if (cnt > 0) {
              tmem_ld32(t_lane + col_acc + c0, v);
              tmem_wait_ld(v);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = 0u;
            }
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float x0 = __uint_as_float(v[e]) * mult, x1 = __uint_as_float(v[e + 1]) * mult;
              if (pb != nullptr) {
                const float* pr = pb + (bh * a.T + rt) * D + c0 + e;
                x0 = fmaf(__ldg(pr), inv_blen, x0);
                x1 = fmaf(__ldg(pr + 1), inv_blen, x1);
              }
              pk[e / 2] = live ? pack_bf16(x0, x1) : 0u;
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_done);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpIssue) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side

constexpr size_t kBwdMaxSmem = 227 * 1024;

template <int R, int D, bool kKeyMajor>
vsa_status launch_bwd_rd(const vsa_plan_s* p, const void* x1, const void* x2, const void* y1,
                         const void* y2, const BwdArgs& a, int64_t bh, cudaStream_t stream) {
  using C = BwdCfg<R, D, kKeyMajor>;
  size_t smem = C::bytes(p->n_tiles) + 1024;
  if (smem < size_t(120 * 1024)) smem = 120 * 1024;   // one CTA per SM: it holds its TMEM
  if (smem > kBwdMaxSmem)
    return fail(VSA_ERR_UNSUPPORTED, "too many tiles for the attention backward kernel's list");
  const int64_t rows = bh * p->n_padded;
  CUtensorMap m1, m2, m3, m4;
  if (!make_map(&m1, x1, rows, D, kBwdM) || !make_map(&m2, x2, rows, D, kBwdM) ||
      !make_map(&m3, y1, rows, D, R) || !make_map(&m4, y2, rows, D, R))
    return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<R, D, kKeyMajor>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, cudaGetErrorString(e));
  const int grid = int(std::min<int64_t>(a.n_items, p->num_sms > 0 ? p->num_sms : 148));
  attn_bwd_kernel<R, D, kKeyMajor><<<grid, kThreadsBwd, smem, stream>>>(m1, m2, m3, m4, a);
  e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(VSA_ERR_CUDA, std::string("attention backward launch: ") + cudaGetErrorString(e));
  return VSA_OK;
}

template <int R, int D>
vsa_status launch_bwd_pair(const vsa_plan_s* p, const void* q_t, const void* k_t, const void* v_t,
                           const void* d_out_t, BwdArgs a, const float* d_qbar, const float* d_kbar,
                           const float* d_vbar, void* dq_t, void* dk_t, void* dv_t, int64_t bh,
                           cudaStream_t stream) {
  // a.next_item holds the two kernels' counters
  unsigned int* const counters = a.next_item;
  // dQ: rows = query tile (Q, dO), columns = its key tiles (K, V)
  a.next_item = counters;
  a.dbar = d_qbar;
  a.dbar2 = nullptr;
  a.out = static_cast<uint16_t*>(dq_t);
  a.out2 = nullptr;
  vsa_status st = launch_bwd_rd<R, D, false>(p, q_t, d_out_t, k_t, v_t, a, bh, stream);
  if (st != VSA_OK) return st;
  // dK, dV: rows = key tile (K, V), columns = the query tiles attending to it (Q, dO)
  a.next_item = counters + 1;
  a.dbar = d_kbar;
  a.dbar2 = d_vbar;
  a.out = static_cast<uint16_t*>(dk_t);
  a.out2 = static_cast<uint16_t*>(dv_t);
  return launch_bwd_rd<R, D, true>(p, k_t, v_t, q_t, d_out_t, a, bh, stream);
}

inline int grid_of(int64_t warps) { return int((warps + 7) / 8); }

}  // namespace

// The attention backward's workspace: the selection bitmap, then the two
// kernels' work counters (16 bytes), all zeroed by one memset per call.
static size_t bitmap_bytes(const vsa_plan_s* p, int64_t bh) {
  const int W = (p->n_tiles + 31) / 32;
  return (size_t(bh) * p->n_tiles * W * 4 + 15) & ~size_t(15);
}

size_t colmask_bytes(const vsa_plan_s* p, int64_t bh) { return bitmap_bytes(p, bh) + 16; }

size_t coarse_bwd_bytes(const vsa_plan_s* p, int64_t bh) {
  return size_t(2) * bh * p->n_tiles * p->n_tiles * 4;
}

cudaError_t launch_combine_backward(const vsa_plan_s* p, const void* d_out_t, const void* o_fine_t,
                                    const void* gate_t, const float* o_coarse, int64_t bh, int D,
                                    float* delta, void* d_gate_t, float* d_oc, cudaStream_t stream) {
  const int64_t items = bh * p->n_tiles;
  if (items == 0) return cudaSuccess;
  auto* dout = static_cast<const uint16_t*>(d_out_t);
  auto* of = static_cast<const uint16_t*>(o_fine_t);
  auto* g = static_cast<const uint16_t*>(gate_t);
  auto* dg = static_cast<uint16_t*>(d_gate_t);
  if (D == 128)
    combine_bwd_kernel<128><<<grid_of(items), 256, 0, stream>>>(dout, of, g, o_coarse, p->d_block_len,
                                                                delta, dg, d_oc, items, p->n_tiles, p->R);
  else
    combine_bwd_kernel<64><<<grid_of(items), 256, 0, stream>>>(dout, of, g, o_coarse, p->d_block_len,
                                                               delta, dg, d_oc, items, p->n_tiles, p->R);
  return cudaGetLastError();
}

cudaError_t launch_coarse_backward(const vsa_plan_s* p, const float* qbar, const float* kbar,
                                   const float* vbar, const float* d_oc, int64_t bh, int D,
                                   float scale, float* d_qbar, float* d_kbar, float* d_vbar,
                                   void* ws, cudaStream_t stream) {
  const int T = p->n_tiles;
  if (bh == 0 || T == 0) return cudaSuccess;
  float* P = static_cast<float*>(ws);
  float* dS = P + bh * int64_t(T) * T;
  const int64_t TD = int64_t(T) * D, TT = int64_t(T) * T;
  auto gemm = [&](const float* A, const float* B, float* Cm, int M, int N, int K, int64_t sab,
                  int64_t sam, int64_t sak, int64_t sbb, int64_t sbk, int64_t sbn, float alpha) {
    dim3 grid((N + kGB - 1) / kGB, (M + kGB - 1) / kGB, unsigned(bh));
    sgemm_kernel<<<grid, 256, 0, stream>>>(A, B, Cm, M, N, K, sab, sam, sak, sbb, sbk, sbn, alpha);
  };
  const int64_t rows = bh * T;
  // P = softmax(scale qbar kbar^T)
  gemm(qbar, kbar, P, T, T, D, TD, D, 1, TD, 1, D, scale);
  softmax_rows_kernel<<<grid_of(rows), 256, 0, stream>>>(P, rows, T);
  // dS = P * (d_oc vbar^T - rowsum)
  gemm(d_oc, vbar, dS, T, T, D, TD, D, 1, TD, 1, D, 1.f);
  softmax_bwd_rows_kernel<<<grid_of(rows), 256, 0, stream>>>(P, dS, rows, T);
  // d_qbar = scale dS kbar;  d_kbar = scale dS^T qbar;  d_vbar = P^T d_oc
  gemm(dS, kbar, d_qbar, T, D, T, TT, T, 1, TD, D, 1, scale);
  gemm(dS, qbar, d_kbar, T, D, T, TT, 1, T, TD, D, 1, scale);
  gemm(P, d_oc, d_vbar, T, D, T, TT, 1, T, TD, D, 1, 1.f);
  return cudaGetLastError();
}

vsa_status launch_sparse_attn_backward(const vsa_plan_s* p, const void* q_t, const void* k_t,
                                       const void* v_t, const void* d_out_t,
                                       const int32_t* topk_idx, int k, const int32_t* topk_ref,
                                       int k_ref, const float* lse_t, const float* delta,
                                       const float* d_qbar, const float* d_kbar,
                                       const float* d_vbar, int64_t bh, int D, float scale,
                                       void* dq_t, void* dk_t, void* dv_t, void* ws,
                                       cudaStream_t stream) {
  if (p->n_padded * bh >= (int64_t(1) << 31))
    return fail(VSA_ERR_UNSUPPORTED, "B*H*N_pad rows exceed the 32-bit TMA coordinate range");
  const int64_t items = bh * p->n_tiles;
  if (items >= (int64_t(1) << 31)) return fail(VSA_ERR_UNSUPPORTED, "too many work items");
  BwdArgs a{};
  a.block_len = p->d_block_len;
  a.topk = topk_idx;
  a.topk_ref = k_ref < 0 ? nullptr : topk_ref;
  a.colmask = static_cast<const uint32_t*>(ws);
  a.next_item = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + bitmap_bytes(p, bh));
  a.lse = lse_t;
  a.delta = delta;
  a.status = p->d_status;
  a.wait_ns = wait_limit_ns();
  a.T = p->n_tiles;
  a.n_p = p->n_prefix_tiles;
  a.k = k;
  a.k_ref = k_ref < 0 ? 0 : k_ref;
  a.n_sink = k_ref < 0 ? p->n_prefix_tiles : k_ref;
  a.W = (p->n_tiles + 31) / 32;
  a.n_items = int(items);
  a.n_pad = p->n_padded;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = cudaMemsetAsync(ws, 0, colmask_bytes(p, bh), stream);
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, std::string("memset: ") + cudaGetErrorString(e));
  colmask_kernel<<<grid_of(items), 256, 0, stream>>>(topk_idx, a.topk_ref, static_cast<uint32_t*>(ws),
                                                     p->d_status, items, a.T, a.n_p, k, a.k_ref,
                                                     a.n_sink, a.W);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, std::string("colmask launch: ") + cudaGetErrorString(e));
  if (p->R == 128) {
    if (D == 128)
      return launch_bwd_pair<128, 128>(p, q_t, k_t, v_t, d_out_t, a, d_qbar, d_kbar, d_vbar, dq_t,
                                       dk_t, dv_t, bh, stream);
    return launch_bwd_pair<128, 64>(p, q_t, k_t, v_t, d_out_t, a, d_qbar, d_kbar, d_vbar, dq_t, dk_t,
                                    dv_t, bh, stream);
  }
  if (D == 128)
    return launch_bwd_pair<64, 128>(p, q_t, k_t, v_t, d_out_t, a, d_qbar, d_kbar, d_vbar, dq_t, dk_t,
                                    dv_t, bh, stream);
  return launch_bwd_pair<64, 64>(p, q_t, k_t, v_t, d_out_t, a, d_qbar, d_kbar, d_vbar, dq_t, dk_t,
                                 dv_t, bh, stream);
}

}  // namespace vsa
