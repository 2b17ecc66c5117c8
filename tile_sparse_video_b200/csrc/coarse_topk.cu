// Coarse attention over pooled tiles and the per-head top-k of video key tiles.
//
// One CTA handles QB = 8*RW query tiles of one (b, h); warp w owns the RW
// query tiles i0 + w*RW ...  The work is three register-tiled fp32 passes:
//   1. scores: s[r][j] = scale * <qbar_r, kbar_j> for all T key tiles.  Key
//      tiles are staged 64 at a time in shared memory (padded rows, so the 32
//      lanes read 32 banks); lane l computes keys l and l+32 for the warp's RW
//      rows, reading the RW query values of one dimension as one broadcast
//      vector load (q is stored transposed).  Scores stay in shared memory.
//   2. top-k (video query tiles only): a radix select over the 32-bit
//      order-preserving image of s[r][j], j in [n_p, T): four 8-bit digit
//      passes with a per-warp 256-bin histogram find the k-th largest key K*;
//      one ascending sweep over j keeps every key > K* and the lowest-index
//      keys == K* until k are kept, which writes the result already sorted by
//      tile index with ties broken towards the lower index.  Bit-exact for
//      given fp32 scores.
//   3. softmax and o_coarse = sum_j p[r][j] vbar_j: the scores become
//      probabilities in place, value tiles are staged 64 at a time, lane l
//      accumulates columns l, l+32, ... for the warp's RW rows.
#include <algorithm>

#include "vsa_internal.h"

namespace vsa {
namespace {

#ifndef VSA_COARSE_KC
#define VSA_COARSE_KC 64
#endif
constexpr int kKC = VSA_COARSE_KC;     // key / value tiles per staged chunk
static_assert(kKC % 32 == 0, "staged chunk: a multiple of 32 tiles");
// Warps per CTA, query rows per warp and CTAs per SM (tuning knobs).
#ifndef VSA_COARSE_WARPS
#define VSA_COARSE_WARPS 8
#endif
#ifndef VSA_COARSE_ROWS
#define VSA_COARSE_ROWS 4
#endif
#ifndef VSA_COARSE_CTAS
#define VSA_COARSE_CTAS 2
#endif
constexpr int kMaxTiles = 4096;        // bound on T (shared-memory budget)

__device__ __forceinline__ uint32_t order_key(float s) {
  s += 0.0f;                                     // -0 -> +0, so equal scores give equal keys
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int RW>
struct QVec;
template <>
struct QVec<1> {
  __device__ static void load(const float* p, float (&q)[1]) { q[0] = p[0]; }
};
template <>
struct QVec<2> {
  __device__ static void load(const float* p, float (&q)[2]) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    q[0] = v.x;
    q[1] = v.y;
  }
};
template <>
struct QVec<4> {
  __device__ static void load(const float* p, float (&q)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    q[0] = v.x;
    q[1] = v.y;
    q[2] = v.z;
    q[3] = v.w;
  }
};

template <>
struct QVec<8> {
  __device__ static void load(const float* p, float (&q)[8]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    const float4 w = *reinterpret_cast<const float4*>(p + 4);
    q[0] = v.x;
    q[1] = v.y;
    q[2] = v.z;
    q[3] = v.w;
    q[4] = w.x;
    q[5] = w.y;
    q[6] = w.z;
    q[7] = w.w;
  }
};

// Asynchronous copy of nj rows of a [*, D] fp32 matrix into a shared-memory
// stage with a padded row stride (D + 4 floats: rows stay 16-byte aligned and
// 128-bit reads of 8 consecutive rows hit 8 distinct bank groups).  One
// commit group per call; the caller waits with cp_async_wait<N>.
template <int D, int kWarps>
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

// Persistent CTAs (two per SM); an item is (b*h, block of QB = NW*RW query
// tiles).  The QB score rows of an item live in this CTA's slot of a global
// scratch area (QB x Tpad fp32, read back from L2), so that QB no longer
// depends on T: every warp keeps RW = 4 query rows in registers against the
// keys it streams from shared memory.
template <int D, int NW, int RW>
__global__ void __launch_bounds__(NW * 32, VSA_COARSE_CTAS) coarse_topk_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, const float* __restrict__ vbar,
    int64_t n_bh, int T, int n_p, float scale, int k, float* __restrict__ o_coarse,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_score, float* __restrict__ scratch) {
  constexpr int kWarps = NW;
  constexpr int QB = kWarps * RW;
  constexpr int kStride = D + 4;
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  float* qT = smem;                                   // [D][QB]; phase 3: P chunk [QB][kKC]
  float* stage0 = qT + D * QB;                        // [2][kKC][kStride]
  uint32_t* hist = reinterpret_cast<uint32_t*>(stage0 + 2 * kKC * kStride);  // [kWarps][256]
  const int Tpad = (T + 3) & ~3;
  float* sc = scratch + int64_t(blockIdx.x) * QB * Tpad;   // this CTA's score rows [QB][Tpad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_blk = (T + QB - 1) / QB;
  const int n_chunks = (T + kKC - 1) / kKC;
  const int n_v = T - n_p;
  const uint32_t lt_mask = (1u << lane) - 1u;

  for (int64_t item = blockIdx.x; item < n_bh * n_blk; item += gridDim.x) {
    const int64_t bh = item / n_blk;
    const int i0 = int(item % n_blk) * QB;
    const float* kb = kbar + bh * int64_t(T) * D;
    const float* vb = vbar + bh * int64_t(T) * D;
    __syncthreads();     // the previous item is done with qT and the stages

    {
      // transposed query block: qT[d][r] (rows past T are zero)
      constexpr int kNVec = QB * D / 4;
      constexpr int kVec = (kNVec + kWarps * 32 - 1) / (kWarps * 32);
      const float4* q4 = reinterpret_cast<const float4*>(qbar + (bh * T + i0) * D);
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int idx = threadIdx.x + u * kWarps * 32;
        if (idx >= kNVec) continue;
        const float4 v = i0 + idx / (D / 4) < T ? __ldg(q4 + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        const int r = idx / (D / 4), d = (idx % (D / 4)) * 4;
        qT[(d + 0) * QB + r] = v.x;
        qT[(d + 1) * QB + r] = v.y;
        qT[(d + 2) * QB + r] = v.z;
        qT[(d + 3) * QB + r] = v.w;
      }
    }

    // ---- 1. scores (double-buffered key stages), written to the scratch rows
    stage_rows_async<D, NW>(stage0, kb, min(kKC, T));
    for (int c = 0; c < n_chunks; ++c) {
      const int j0 = c * kKC;
      const int nj = min(kKC, T - j0);
      float* stage = stage0 + (c & 1) * kKC * kStride;
      if (c + 1 < n_chunks) {
        stage_rows_async<D, NW>(stage0 + ((c + 1) & 1) * kKC * kStride, kb + int64_t(j0 + kKC) * D,
                                min(kKC, T - j0 - kKC));
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      constexpr int KPL = kKC / 32;                  // keys per lane: lane, lane + 32, ...
      float acc[RW][KPL];
#pragma unroll
      for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int u = 0; u < KPL; ++u) acc[r][u] = 0.f;
      const float* qw = qT + warp * RW;
#pragma unroll 4
      for (int d4 = 0; d4 < D / 4; ++d4) {
        float av[KPL][4];
#pragma unroll
        for (int u = 0; u < KPL; ++u) {
          const float4 a = reinterpret_cast<const float4*>(stage + (lane + 32 * u) * kStride)[d4];
          av[u][0] = a.x;
          av[u][1] = a.y;
          av[u][2] = a.z;
          av[u][3] = a.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float q[RW];
          QVec<RW>::load(qw + (4 * d4 + e) * QB, q);
#pragma unroll
          for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int u = 0; u < KPL; ++u) acc[r][u] = fmaf(q[r], av[u][e], acc[r][u]);
        }
      }
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        float* row = sc + (warp * RW + r) * Tpad + j0;
#pragma unroll
        for (int u = 0; u < KPL; ++u)
          if (lane + 32 * u < nj) row[lane + 32 * u] = scale * acc[r][u];
      }
      __syncthreads();     // stage (c & 1) is refilled two chunks later
    }

    // ---- 2. per row of this warp: the scores copied from the scratch row
    // into a shared-memory row buffer of the warp (in the key stages, free
    // now) when they fit, then the top-k over the video key tiles (video
    // query tiles only) and the softmax, whose P goes back to the scratch row
    uint32_t* h = hist + warp * 256;
    const bool row_in_smem = size_t(kWarps) * Tpad <= size_t(2) * kKC * kStride;
    float inv_l[RW];
    for (int r = 0; r < RW; ++r) {
      const int i = i0 + warp * RW + r;
      float* srow = sc + (warp * RW + r) * Tpad;                 // global
      float* s = row_in_smem ? stage0 + warp * Tpad : srow;     // where the passes read
      if (row_in_smem) {
        for (int j4 = lane; j4 < Tpad / 4; j4 += 32)
          reinterpret_cast<float4*>(s)[j4] = reinterpret_cast<const float4*>(srow)[j4];
        __syncwarp();
      }
      if (i < T && i >= n_p && k > 0) {
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
        // prefix = K*, remaining = number of keys equal to K* to keep (lowest j first)
        int32_t* out_idx = topk_idx + ((bh * n_v) + (i - n_p)) * int64_t(k);
        float* out_s = topk_score ? topk_score + ((bh * n_v) + (i - n_p)) * int64_t(k) : nullptr;
        int pos = 0, eq_seen = 0;
        for (int base = n_p; base < T; base += 32) {
          const int j = base + lane;
          const bool valid = j < T;
          const float sv = valid ? s[j] : 0.f;
          const uint32_t key = valid ? order_key(sv) : 0u;
          const bool gt = valid && key > prefix;
          const bool eq = valid && key == prefix;
          const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
          const int eq_rank = eq_seen + __popc(eqb & lt_mask);
          const bool sel = gt || (eq && eq_rank < remaining);
          const uint32_t selb = __ballot_sync(0xFFFFFFFFu, sel);
          if (sel) {
            const int o = pos + __popc(selb & lt_mask);
            out_idx[o] = j;
            if (out_s) out_s[o] = sv;
          }
          pos += __popc(selb);
          eq_seen += __popc(eqb);
        }
      }
      // ---- 3a. softmax of the row; P to the scratch row
      float m = -INFINITY;
      for (int j = lane; j < T; j += 32) m = fmaxf(m, s[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      float l = 0.f;
      for (int j = lane; j < T; j += 32) {
        const float p = __expf(s[j] - m);
        srow[j] = p;
        l += p;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
      inv_l[r] = 1.0f / l;
      __syncwarp();        // the row buffer is refilled for the next row
    }

    // ---- 3b. o_coarse = P V / l: P chunks staged into shared memory next to
    // the value chunks
    float acc[RW][D / 32];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < D / 32; ++c) acc[r][c] = 0.f;
    __syncthreads();     // every P row written; qT no longer needed (P stage)
    float* pst = qT;     // [2][QB][kKC]
    auto stage_p = [&](int buf, int j0, int nj) {
      // P[r][j0 .. j0 + nj) of all QB rows; 16-byte pieces (j0 and Tpad are
      // multiples of 4; a ragged tail piece reads past nj into the row's
      // padding, never past the scratch slot)
      constexpr int kPieces = QB * (kKC / 4);
      for (int idx = threadIdx.x; idx < kPieces; idx += kWarps * 32) {
        const int r = idx / (kKC / 4), q4 = (idx % (kKC / 4)) * 4;
        if (q4 >= nj) continue;
        const uint32_t dst = static_cast<uint32_t>(
            __cvta_generic_to_shared(pst + buf * QB * kKC + r * kKC + q4));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                     "l"(sc + r * Tpad + j0 + q4)
                     : "memory");
      }
    };
    stage_p(0, 0, min(kKC, T));
    stage_rows_async<D, NW>(stage0, vb, min(kKC, T));
    for (int c = 0; c < n_chunks; ++c) {
      const int j0 = c * kKC;
      const int nj = min(kKC, T - j0);
      const float* stage = stage0 + (c & 1) * kKC * kStride;
      const float* pc = pst + (c & 1) * QB * kKC;
      if (c + 1 < n_chunks) {
        stage_p((c + 1) & 1, j0 + kKC, min(kKC, T - j0 - kKC));
        stage_rows_async<D, NW>(stage0 + ((c + 1) & 1) * kKC * kStride, vb + int64_t(j0 + kKC) * D,
                                min(kKC, T - j0 - kKC));
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      for (int jj = 0; jj < nj; ++jj) {
        float v[D / 32];
#pragma unroll
        for (int c2 = 0; c2 < D / 32; ++c2) v[c2] = stage[jj * kStride + lane + 32 * c2];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          const float p = pc[(warp * RW + r) * kKC + jj];
#pragma unroll
          for (int c2 = 0; c2 < D / 32; ++c2) acc[r][c2] = fmaf(p, v[c2], acc[r][c2]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int i = i0 + warp * RW + r;
      if (i >= T) continue;
      float* oc = o_coarse + (bh * T + i) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) oc[lane + 32 * c] = acc[r][c] * inv_l[r];
    }
  }
}

constexpr int kCoarseWarps = VSA_COARSE_WARPS, kCoarseRows = VSA_COARSE_ROWS;   // QB = 32 query tiles per item
constexpr int kCoarseQB = kCoarseWarps * kCoarseRows;

template <int D>
size_t coarse_smem_bytes() {
  // qT [D][QB] (reused as two P stages [QB][kKC]), two key / value stages,
  // the per-warp histograms
  const size_t q = size_t(D) * kCoarseQB;
  const size_t p = size_t(2) * kCoarseQB * kKC;
  return sizeof(float) * ((q > p ? q : p) + size_t(2) * kKC * (D + 4) + size_t(kCoarseWarps) * 256);
}

template <int D>
cudaError_t launch_coarse_d(const float* qbar, const float* kbar, const float* vbar, int64_t bh,
                            int T, int n_p, float scale, int k, float* o_coarse, int32_t* topk_idx,
                            float* topk_score, float* scratch, int grid, cudaStream_t stream) {
  const size_t smem = coarse_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(coarse_topk_kernel<D, kCoarseWarps, kCoarseRows>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  coarse_topk_kernel<D, kCoarseWarps, kCoarseRows><<<grid, kCoarseWarps * 32, smem, stream>>>(
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
  return sizeof(float) * size_t(coarse_grid(num_sms)) * kCoarseQB * size_t((T + 3) & ~3);
}

cudaError_t launch_coarse_topk(const float* qbar, const float* kbar, const float* vbar, int64_t bh,
                               int T, int n_p, int D, float scale, int k, float* o_coarse,
                               int32_t* topk_idx, float* topk_score, float* scratch, int num_sms,
                               cudaStream_t stream) {
  if (T > kMaxTiles) return cudaErrorInvalidValue;
  const int64_t items = bh * ((T + kCoarseQB - 1) / kCoarseQB);
  if (items == 0) return cudaSuccess;
  const int grid = int(std::min<int64_t>(items, coarse_grid(num_sms)));
  if (D == 128)
    return launch_coarse_d<128>(qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx,
                                topk_score, scratch, grid, stream);
  return launch_coarse_d<64>(qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx,
                             topk_score, scratch, grid, stream);
}

}  // namespace vsa
