// Coarse attention over pooled tiles and the per-head top-k of video key tiles.
//
// Persistent CTAs (two per SM, eight warps); an item is (b*h, block of QB = 32
// query tiles).  The QB score rows of an item live in this CTA's slot of a
// global scratch area (QB x ceil4(T) fp32, which stays in L2), so the block
// size does not depend on T.  Three passes per item:
//   1. scores: s[r][j] = scale * <qbar_r, kbar_j> for all T key tiles, fp32
//      FMAs in ascending d.  Key tiles are staged 64 at a time in shared
//      memory; lane (rg, kg) of warp w computes rows rg + 8i (i < 4) against
//      keys 8w + 2kg + {0, 1}, so that every shared-memory read of a warp is a
//      broadcast of at most eight distinct 16-byte words (one wavefront).
//   2. per row (a warp takes four): the row max, then the top-k over the
//      video key tiles (video query tiles only).  A histogram over the row's
//      value range (256 equal-width bins of (s - min) * 256 / (max - min), a
//      monotone map of s) finds the bin that holds the k-th largest score; its
//      scores (at most 32; else, and for a row holding a NaN score, the exact
//      radix select below runs instead) are ranked against each other, which
//      gives the k-th largest score K* and how many scores equal to K* to keep.  One ascending sweep then keeps every
//      score > K* and the lowest-index scores == K*, so the result is sorted by
//      tile index with ties broken towards the lower index; bit-exact for given
//      fp32 scores.  The fallback radix select runs four 8-bit digit passes
//      over the 32-bit order-preserving image of s.
//   3. o_coarse = softmax(s) vbar: the probabilities p = exp(s - max) are made
//      while staging, 64 key tiles at a time, next to the value tiles; lane
//      (rg, cg) accumulates rows rg + 8i against D/32 consecutive columns, and
//      the row sums of p in the same loop.
#include <algorithm>

#include "vsa_internal.h"

namespace vsa {
namespace {

#ifndef VSA_COARSE_KC
#define VSA_COARSE_KC 64
#endif
constexpr int kKC = VSA_COARSE_KC;     // key / value tiles per staged chunk
static_assert(kKC == 64, "the lane maps below cover 64 key tiles per chunk");
// CTAs per SM (tuning knob).
#ifndef VSA_COARSE_CTAS
#define VSA_COARSE_CTAS 2
#endif
constexpr int kWarps = 8;
constexpr int kQB = 32;                // query tiles per item: 8 row groups x 4
constexpr int kRowsPerWarp = kQB / kWarps;
constexpr int kPStride = kKC + 4;      // row stride of a staged probability chunk
constexpr int kMaxTiles = 4096;        // bound on T (shared-memory budget)

__device__ __forceinline__ uint32_t order_key(float s) {
  s += 0.0f;                                     // -0 -> +0, so equal scores give equal keys
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Asynchronous copy of nj rows of a [*, D] fp32 matrix into a shared-memory
// stage with a padded row stride (D + 4 floats: rows stay 16-byte aligned and
// 128-bit reads of 8 consecutive rows hit 8 distinct bank groups).  One
// commit group per call; the caller waits with cp_async_wait<N>.
template <int D>
__device__ __forceinline__ void stage_rows_async(float* stage, const float* src, int nj) {
  constexpr int kStride = D + 4;
  constexpr int kVecPerRow = D / 4;
  constexpr int kPerThread = (kKC * kVecPerRow) / (kWarps * 32);
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int idx = threadIdx.x + u * kWarps * 32;
    if (idx < nj * kVecPerRow) {
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(
          stage + (idx / kVecPerRow) * kStride + (idx % kVecPerRow) * 4));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + idx * 4)
                   : "memory");
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Exact radix select of the k-th largest order key over s[n_p, T) (one warp):
// four 8-bit digit passes, each a histogram of the digit among the keys that
// match the digits chosen so far.  Returns (K*, number of keys equal to K* to
// keep).  Out of line: it runs only when the range histogram cannot isolate
// the k-th score.
__device__ __noinline__ uint2 radix_select(const float* s, int T, int n_p, int k, uint32_t* h,
                                           int lane) {
  uint32_t prefix = 0u, mask = 0u;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int b = 0; b < 8; ++b) h[lane * 8 + b] = 0u;
    __syncwarp();
    for (int jb = n_p; jb < T; jb += 32) {
      const int j = jb + lane;
      const uint32_t key = j < T ? order_key(s[j]) : 0u;
      const bool in = j < T && (key & mask) == prefix;
      // lanes with the same digit add once (scores cluster in few bins)
      const uint32_t bin = in ? ((key >> shift) & 255u) : 256u;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
      if (in && (__ffs(peers) - 1) == lane) atomicAdd(h + bin, uint32_t(__popc(peers)));
    }
    __syncwarp();
    // lane L holds bins 255-8L .. 248-8L (lane 0 = highest digits)
    uint32_t cnt = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) cnt += h[255 - 8 * lane - b];
    uint32_t incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += o;
    }
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, incl >= uint32_t(remaining));
    const int L = __ffs(ballot) - 1;
    uint32_t digit = 0;
    int rem_new = 0;
    if (lane == L) {
      uint32_t run = incl - cnt;                      // keys with a higher digit
      for (int b = 0; b < 8; ++b) {
        const uint32_t bin = 255 - 8 * L - b;
        if (run + h[bin] >= uint32_t(remaining)) {
          digit = bin;
          rem_new = remaining - int(run);
          break;
        }
        run += h[bin];
      }
    }
    digit = __shfl_sync(0xFFFFFFFFu, digit, L);
    remaining = __shfl_sync(0xFFFFFFFFu, rem_new, L);
    prefix |= digit << shift;
    mask |= 255u << shift;
    __syncwarp();
  }
  return make_uint2(prefix, uint32_t(remaining));
}

// Range-histogram bin of a score: floor((s - lo) * sc) clamped to [0, 255]
// (monotone non-decreasing in s: a larger score never lands in a lower bin).
__device__ __forceinline__ int range_bin(float s, float lo, float sc) {
  return int(fminf(fmaxf((s - lo) * sc, 0.0f), 255.0f));
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32, VSA_COARSE_CTAS) coarse_topk_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, const float* __restrict__ vbar,
    int64_t n_bh, int T, int n_p, float scale, int k, float* __restrict__ o_coarse,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_score, float* __restrict__ scratch) {
  constexpr int kStride = D + 4;
  constexpr int CPL = D / 32;                 // output columns per lane in pass 3
  constexpr int kQFloats = D * kQB, kPFloats = 2 * kQB * kPStride;
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  // qT [D][QB] in pass 1, the two probability stages [2][QB][kPStride] in pass 3
  float* qT = smem;
  float* stage0 = qT + (kQFloats > kPFloats ? kQFloats : kPFloats);   // [2][kKC][kStride]
  uint32_t* hist = reinterpret_cast<uint32_t*>(stage0 + 2 * kKC * kStride);   // [kWarps][256]
  uint32_t* cand = hist + kWarps * 256;                                       // [kWarps][32]
  float* row_max = reinterpret_cast<float*>(cand + kWarps * 32);              // [QB]
  const int Tpad = (T + 3) & ~3;
  float* sc = scratch + int64_t(blockIdx.x) * kQB * Tpad;   // this CTA's score rows [QB][Tpad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane >> 2, sub = lane & 3;   // row group (rows rg + 8i), key / column group
  const int n_blk = (T + kQB - 1) / kQB;
  const int n_chunks = (T + kKC - 1) / kKC;
  const int n_v = T - n_p;
  const uint32_t lt_mask = (1u << lane) - 1u;

  for (int64_t item = blockIdx.x; item < n_bh * n_blk; item += gridDim.x) {
    const int64_t bh = item / n_blk;
    const int i0 = int(item % n_blk) * kQB;
    const float* kb = kbar + bh * int64_t(T) * D;
    const float* vb = vbar + bh * int64_t(T) * D;
    __syncthreads();     // the previous item is done with every shared buffer

    {
      // transposed query block: qT[d][4 * (r % 8) + r / 8] (rows past T are zero),
      // so that a lane's four rows rg + 8i are one 16-byte word per dimension
      constexpr int kNVec = kQB * D / 4;
      const float4* q4 = reinterpret_cast<const float4*>(qbar + (bh * T + i0) * D);
      for (int idx = threadIdx.x; idx < kNVec; idx += kWarps * 32) {
        const int r = idx / (D / 4), d = (idx % (D / 4)) * 4;
        const float4 v = i0 + r < T ? __ldg(q4 + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        const int pos = 4 * (r & 7) + (r >> 3);
        qT[(d + 0) * kQB + pos] = v.x;
        qT[(d + 1) * kQB + pos] = v.y;
        qT[(d + 2) * kQB + pos] = v.z;
        qT[(d + 3) * kQB + pos] = v.w;
      }
    }

    // ---- 1. scores (double-buffered key stages), written to the scratch rows
    stage_rows_async<D>(stage0, kb, min(kKC, T));
    for (int c = 0; c < n_chunks; ++c) {
      const int j0 = c * kKC;
      const int nj = min(kKC, T - j0);
      const float* stage = stage0 + (c & 1) * kKC * kStride;
      if (c + 1 < n_chunks) {
        stage_rows_async<D>(stage0 + ((c + 1) & 1) * kKC * kStride, kb + int64_t(j0 + kKC) * D,
                            min(kKC, T - j0 - kKC));
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const int jl = 8 * warp + 2 * sub;             // this lane's two keys: jl, jl + 1
      float acc[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.f;
      const float* k0 = stage + jl * kStride;
      const float* qg = qT + 4 * rg;
#pragma unroll 4
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 a = reinterpret_cast<const float4*>(k0)[d4];
        const float4 b = reinterpret_cast<const float4*>(k0 + kStride)[d4];
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 q = *reinterpret_cast<const float4*>(qg + (4 * d4 + e) * kQB);
          const float qv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[i][0] = fmaf(qv[i], av[e], acc[i][0]);
            acc[i][1] = fmaf(qv[i], bv[e], acc[i][1]);
          }
        }
      }
      if (jl < nj) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float* row = sc + (rg + 8 * i) * Tpad + j0 + jl;
          if (jl + 1 < nj)
            *reinterpret_cast<float2*>(row) = make_float2(scale * acc[i][0], scale * acc[i][1]);
          else
            row[0] = scale * acc[i][0];
        }
      }
      __syncthreads();     // stage (c & 1) is refilled two chunks later
    }

    // ---- 2. per row of this warp: the row max (for the softmax) and, for
    // video query tiles, the top-k over the video key tiles.  The row is
    // copied from the scratch into a shared-memory row buffer of the warp (in
    // the key stages, free now) when it fits.
    uint32_t* h = hist + warp * 256;
    uint32_t* cw = cand + warp * 32;
    const bool row_in_smem = size_t(kWarps) * Tpad <= size_t(2) * kKC * kStride;
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = warp * kRowsPerWarp + rr;
      const int i = i0 + r;
      const float* srow = sc + r * Tpad;                         // global
      const float* s = srow;
      if (row_in_smem) {
        float* buf = stage0 + warp * Tpad;
        for (int j4 = lane; j4 < Tpad / 4; j4 += 32)
          reinterpret_cast<float4*>(buf)[j4] = reinterpret_cast<const float4*>(srow)[j4];
        __syncwarp();
        s = buf;
      }
      // row max over all T tiles; min and max over the video tiles, and
      // whether one of them is NaN (the range histogram would bin it apart
      // from where its order key ranks it, so such rows take the radix select)
      float m = -INFINITY, vlo = INFINITY, vhi = -INFINITY;
      bool nan_seen = false;
#pragma unroll 2
      for (int j = lane; j < T; j += 32) {
        const float v = s[j];
        m = fmaxf(m, v);
        if (j >= n_p) {
          vlo = fminf(vlo, v);
          vhi = fmaxf(vhi, v);
          nan_seen |= v != v;
        }
      }
      const bool row_nan = __any_sync(0xFFFFFFFFu, nan_seen);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        vlo = fminf(vlo, __shfl_xor_sync(0xFFFFFFFFu, vlo, off));
        vhi = fmaxf(vhi, __shfl_xor_sync(0xFFFFFFFFu, vhi, off));
      }
      if (lane == 0) row_max[r] = i < T ? m : 0.f;
      if (i < T && i >= n_p && k > 0) {
        uint32_t kstar = 0u;
        int remaining = 0;
        bool found = false;
        const float range = vhi - vlo;
        const float bsc = 256.0f / range;
        if (!row_nan && range > 0.0f && range < INFINITY && bsc < INFINITY) {
          // one histogram over the value range
#pragma unroll
          for (int b = 0; b < 8; ++b) h[lane * 8 + b] = 0u;
          __syncwarp();
#pragma unroll 2
          for (int j = n_p + lane; j < T; j += 32) atomicAdd(h + range_bin(s[j], vlo, bsc), 1u);
          __syncwarp();
          // lane L holds bins 255-8L .. 248-8L (lane 0 = highest scores)
          uint32_t cnt = 0;
#pragma unroll
          for (int b = 0; b < 8; ++b) cnt += h[255 - 8 * lane - b];
          uint32_t incl = cnt;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += o;
          }
          const int L = __ffs(__ballot_sync(0xFFFFFFFFu, incl >= uint32_t(k))) - 1;
          int bstar = 0, above = 0, in_bin = 0;
          if (lane == L) {
            uint32_t run = incl - cnt;                  // scores in higher bins
            for (int b = 0; b < 8; ++b) {
              const int bin = 255 - 8 * L - b;
              if (run + h[bin] >= uint32_t(k)) {
                bstar = bin;
                above = int(run);
                in_bin = int(h[bin]);
                break;
              }
              run += h[bin];
            }
          }
          bstar = __shfl_sync(0xFFFFFFFFu, bstar, L);
          above = __shfl_sync(0xFFFFFFFFu, above, L);
          in_bin = __shfl_sync(0xFFFFFFFFu, in_bin, L);
          if (in_bin <= 32) {
            // the scores of bin b*, compacted; the k-th largest is among them
            int base = 0;
#pragma unroll 2
            for (int jb = n_p; jb < T; jb += 32) {
              const int j = jb + lane;
              const float v = j < T ? s[j] : 0.f;
              const bool in = j < T && range_bin(v, vlo, bsc) == bstar;
              const uint32_t b = __ballot_sync(0xFFFFFFFFu, in);
              if (in) cw[base + __popc(b & lt_mask)] = order_key(v);
              base += __popc(b);
            }
            __syncwarp();
            const int need = k - above;                 // 1 <= need <= in_bin
            uint32_t key = 0u;
            int gt = 0, eq = 0;
            if (lane < in_bin) {
              key = cw[lane];
              for (int u = 0; u < in_bin; ++u) {
                const uint32_t o = cw[u];
                gt += o > key ? 1 : 0;
                eq += o == key ? 1 : 0;
              }
            }
            const uint32_t hit = __ballot_sync(0xFFFFFFFFu, lane < in_bin && gt < need && need <= gt + eq);
            if (hit != 0u) {
              const int L2 = __ffs(hit) - 1;
              kstar = __shfl_sync(0xFFFFFFFFu, key, L2);
              remaining = need - __shfl_sync(0xFFFFFFFFu, gt, L2);
              found = true;
            }
            __syncwarp();
          }
        }
        if (!found) {
          const uint2 sel = radix_select(s, T, n_p, k, h, lane);
          kstar = sel.x;
          remaining = int(sel.y);
        }
        // keep every key > K* and the lowest-index `remaining` keys == K*
        int32_t* out_idx = topk_idx + ((bh * n_v) + (i - n_p)) * int64_t(k);
        float* out_s = topk_score ? topk_score + ((bh * n_v) + (i - n_p)) * int64_t(k) : nullptr;
        int pos = 0, eq_seen = 0;
#pragma unroll 2
        for (int base = n_p; base < T; base += 32) {
          const int j = base + lane;
          const bool valid = j < T;
          const float sv = valid ? s[j] : 0.f;
          const uint32_t key = valid ? order_key(sv) : 0u;
          const bool gt = valid && key > kstar;
          const bool eq = valid && key == kstar;
          const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
          const int eq_rank = eq_seen + __popc(eqb & lt_mask);
          const bool sel = gt || (eq && eq_rank < remaining);
          const uint32_t selb = __ballot_sync(0xFFFFFFFFu, sel);
          if (sel) {
            const int o = pos + __popc(selb & lt_mask);
            if (o < k) {             // exactly k are selected; the bound only guards the row
              out_idx[o] = j;
              if (out_s) out_s[o] = sv;
            }
          }
          pos += __popc(selb);
          eq_seen += __popc(eqb);
        }
      }
      __syncwarp();        // the row buffer is refilled for the next row
    }

    // ---- 3. o_coarse = sum_j p[r][j] vbar_j / sum_j p[r][j], p = exp(s - max):
    // p made while staging (thread t: row t / 8, eight tiles from 8 (t % 8)),
    // value chunks staged by cp.async beside them
    __syncthreads();     // row maxima written; qT and the row buffers free
    float* pst = qT;     // [2][QB][kPStride]
    const int pr_row = threadIdx.x >> 3, pr_col = (threadIdx.x & 7) * 8;
    float pv[8];
    auto load_p = [&](int j0) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int j = j0 + pr_col + 4 * hh;
        const float4 v = j < Tpad ? *reinterpret_cast<const float4*>(sc + pr_row * Tpad + j)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        pv[4 * hh + 0] = v.x;
        pv[4 * hh + 1] = v.y;
        pv[4 * hh + 2] = v.z;
        pv[4 * hh + 3] = v.w;
      }
    };
    auto store_p = [&](int buf, int j0) {
      const float mr = row_max[pr_row];
      float e[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) e[u] = j0 + pr_col + u < T ? __expf(pv[u] - mr) : 0.f;
      float4* dst = reinterpret_cast<float4*>(pst + buf * kQB * kPStride + pr_row * kPStride + pr_col);
      dst[0] = make_float4(e[0], e[1], e[2], e[3]);
      dst[1] = make_float4(e[4], e[5], e[6], e[7]);
    };
    const int c0 = warp * 4 * CPL + sub * CPL;   // this lane's output columns
    float acc[4][CPL], lsum[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lsum[i] = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[i][c] = 0.f;
    }
    load_p(0);
    store_p(0, 0);
    stage_rows_async<D>(stage0, vb, min(kKC, T));
    for (int c = 0; c < n_chunks; ++c) {
      const int j0 = c * kKC;
      const int nj = min(kKC, T - j0);
      const float* stage = stage0 + (c & 1) * kKC * kStride;
      const float* pc = pst + (c & 1) * kQB * kPStride;
      if (c + 1 < n_chunks) {
        stage_rows_async<D>(stage0 + ((c + 1) & 1) * kKC * kStride, vb + int64_t(j0 + kKC) * D,
                            min(kKC, T - j0 - kKC));
        load_p(j0 + kKC);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();     // value chunk c landed, probability chunk c stored
      const float* pr = pc + rg * kPStride;
      const int nj4 = nj & ~3;
#pragma unroll 4
      for (int jj = 0; jj < nj4; jj += 4) {
        float p[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 t = *reinterpret_cast<const float4*>(pr + 8 * i * kPStride + jj);
          p[i][0] = t.x;
          p[i][1] = t.y;
          p[i][2] = t.z;
          p[i][3] = t.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v[CPL];
          if constexpr (CPL == 4) {
            const float4 t = *reinterpret_cast<const float4*>(stage + (jj + e) * kStride + c0);
            v[0] = t.x;
            v[1] = t.y;
            v[2] = t.z;
            v[3] = t.w;
          } else {
            const float2 t = *reinterpret_cast<const float2*>(stage + (jj + e) * kStride + c0);
            v[0] = t.x;
            v[1] = t.y;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            lsum[i] += p[i][e];
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) acc[i][cc] = fmaf(p[i][e], v[cc], acc[i][cc]);
          }
        }
      }
      for (int jj = nj4; jj < nj; ++jj) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float pp = pr[8 * i * kPStride + jj];
          lsum[i] += pp;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc)
            acc[i][cc] = fmaf(pp, stage[jj * kStride + c0 + cc], acc[i][cc]);
        }
      }
      if (c + 1 < n_chunks) store_p((c + 1) & 1, j0 + kKC);
      __syncthreads();     // both stages of chunk c are refilled one chunk later
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = rg + 8 * i;
      if (i0 + r >= T) continue;
      float* oc = o_coarse + (bh * T + i0 + r) * D + c0;
      const float inv = 1.0f / lsum[i];
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) oc[cc] = acc[i][cc] * inv;
    }
  }
}

template <int D>
size_t coarse_smem_bytes() {
  // qT [D][QB] (reused as two probability stages [QB][kPStride]), two key /
  // value stages, the per-warp histograms and candidate lists, the row maxima
  const size_t q = size_t(D) * kQB;
  const size_t p = size_t(2) * kQB * kPStride;
  return sizeof(float) * ((q > p ? q : p) + size_t(2) * kKC * (D + 4) + size_t(kWarps) * (256 + 32) +
                          kQB);
}

template <int D>
cudaError_t launch_coarse_d(const float* qbar, const float* kbar, const float* vbar, int64_t bh,
                            int T, int n_p, float scale, int k, float* o_coarse, int32_t* topk_idx,
                            float* topk_score, float* scratch, int grid, cudaStream_t stream) {
  const size_t smem = coarse_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(coarse_topk_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  coarse_topk_kernel<D><<<grid, kWarps * 32, smem, stream>>>(
      qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx, topk_score, scratch);
  return cudaGetLastError();
}

// Reference-tile selection (the Veda node's reference_sparsity): for every
// video query tile i (n_p <= i < T) of every (b, h), the k_ref reference key
// tiles j < n_p with the largest s[i,j] = scale * <qbar_i, kbar_j>, ties to
// the lower j, written ascending to out[bh, i - n_p, :].  One warp per row:
// lane-strided fp32 dot products (d ascending, the order the coarse kernel
// uses, so the scores are the same bits) into a shared row of n_p scores;
// then every candidate's rank by counting the keys that beat it (a larger
// score, or an equal one at a lower index), and a ballot prefix count of the
// kept ones for the ascending output.
constexpr int kRefMaxTiles = 256;
constexpr int kRefWarps = 8;

template <int D>
__global__ void __launch_bounds__(kRefWarps * 32) select_ref_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, int64_t n_rows, int T, int n_p,
    float scale, int k_ref, int32_t* __restrict__ out) {
  __shared__ float sc[kRefWarps][kRefMaxTiles];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_v = T - n_p;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int64_t r = int64_t(blockIdx.x) * kRefWarps + warp; r < n_rows;
       r += int64_t(gridDim.x) * kRefWarps) {
    const int64_t bh = r / n_v;
    const int i = n_p + int(r % n_v);
    const float4* q4 = reinterpret_cast<const float4*>(qbar + (bh * T + i) * D);
    for (int j = lane; j < n_p; j += 32) {
      const float4* k4 = reinterpret_cast<const float4*>(kbar + (bh * T + j) * D);
      float acc = 0.f;
#pragma unroll 8
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 a = __ldg(q4 + d4), b = __ldg(k4 + d4);
        acc = fmaf(a.x, b.x, acc);
        acc = fmaf(a.y, b.y, acc);
        acc = fmaf(a.z, b.z, acc);
        acc = fmaf(a.w, b.w, acc);
      }
      sc[warp][j] = scale * acc;
    }
    __syncwarp();
    int32_t* o = out + r * k_ref;
    int base = 0;
    for (int j0 = 0; j0 < n_p; j0 += 32) {
      const int j = j0 + lane;
      bool keep = false;
      if (j < n_p) {
        const float sj = sc[warp][j];
        int rank = 0;
        for (int m = 0; m < n_p; ++m) {
          const float sm = sc[warp][m];
          rank += (sm > sj || (sm == sj && m < j)) ? 1 : 0;
        }
        keep = rank < k_ref;
      }
      const uint32_t b = __ballot_sync(0xFFFFFFFFu, keep);
      const int pos = base + __popc(b & lt_mask);
      if (keep && pos < k_ref) o[pos] = j;      // exactly k_ref keep for finite scores
      base += __popc(b);
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_select_ref(const float* qbar, const float* kbar, int64_t bh, int T, int n_p, int D,
                              float scale, int k_ref, int32_t* topk_ref, int num_sms,
                              cudaStream_t stream) {
  if (n_p > kRefMaxTiles) return cudaErrorInvalidValue;
  const int64_t n_rows = bh * (T - n_p);
  if (n_rows == 0 || k_ref == 0) return cudaSuccess;
  int64_t blocks = (n_rows + kRefWarps - 1) / kRefWarps;
  const int64_t cap = int64_t(num_sms > 0 ? num_sms : 148) * 8;
  if (blocks > cap) blocks = cap;
  if (D == 128)
    select_ref_kernel<128><<<unsigned(blocks), kRefWarps * 32, 0, stream>>>(qbar, kbar, n_rows, T, n_p,
                                                                             scale, k_ref, topk_ref);
  else
    select_ref_kernel<64><<<unsigned(blocks), kRefWarps * 32, 0, stream>>>(qbar, kbar, n_rows, T, n_p,
                                                                            scale, k_ref, topk_ref);
  return cudaGetLastError();
}

int coarse_grid(int num_sms) { return VSA_COARSE_CTAS * (num_sms > 0 ? num_sms : 148); }

size_t coarse_scratch_bytes(int T, int num_sms) {
  return sizeof(float) * size_t(coarse_grid(num_sms)) * kQB * size_t((T + 3) & ~3);
}

cudaError_t launch_coarse_topk(const float* qbar, const float* kbar, const float* vbar, int64_t bh,
                               int T, int n_p, int D, float scale, int k, float* o_coarse,
                               int32_t* topk_idx, float* topk_score, float* scratch, int num_sms,
                               cudaStream_t stream) {
  if (T > kMaxTiles) return cudaErrorInvalidValue;
  const int64_t items = bh * ((T + kQB - 1) / kQB);
  if (items == 0) return cudaSuccess;
  const int grid = int(std::min<int64_t>(items, coarse_grid(num_sms)));
  if (D == 128)
    return launch_coarse_d<128>(qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx,
                                topk_score, scratch, grid, stream);
  return launch_coarse_d<64>(qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx,
                             topk_score, scratch, grid, stream);
}

}  // namespace vsa
