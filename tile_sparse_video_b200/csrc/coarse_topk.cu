// Coarse attention over pooled tiles and the per-head top-k of video key tiles.
//
// One CTA of kQB warps handles kQB query tiles of one (b, h); warp w owns query
// tile i0 + w.  Pooled key (then value) tiles are staged through shared memory
// in chunks of 32, shared by the kQB warps.  Per warp:
//   1. s[j] = scale * <qbar_i, kbar_j> for all T key tiles (lane = key tile of
//      the chunk; the staging buffer has a padded row stride so the 32 lanes
//      read 32 different banks), kept in shared memory in fp32;
//   2. o_coarse_i = sum_j softmax(s)_j vbar_j (lane = 4 output columns);
//   3. for a video query tile, a radix select over the 32-bit order-preserving
//      image of s[j], j in [n_p, T): four 8-bit digit passes with a per-warp
//      256-bin histogram find the k-th largest key K*; then one ascending sweep
//      over j keeps every key > K* and the lowest-index keys == K* until k are
//      kept, which writes the result already sorted by tile index and breaks
//      ties towards the lower index.  Bit-exact for given fp32 scores.
#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kQB = 8;                 // query tiles (= warps) per CTA
constexpr int kKC = 32;                // key tiles per staged chunk
constexpr int kMaxTiles = 4096;        // bound on T (shared-memory budget)

__device__ __forceinline__ uint32_t order_key(float s) {
  s += 0.0f;                                     // -0 -> +0, so equal scores give equal keys
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D>
__global__ void __launch_bounds__(kQB * 32) coarse_topk_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, const float* __restrict__ vbar,
    int T, int n_p, float scale, int k, float* __restrict__ o_coarse, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_score) {
  constexpr int kStride = D + 1;
  extern __shared__ float smem[];
  float* stage = smem;                           // [kKC][kStride]
  float* qrow = stage + kKC * kStride;           // [kQB][D]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qrow + kQB * D);   // [kQB][256]
  float* srow = reinterpret_cast<float*>(hist + kQB * 256);       // [kQB][Tpad]
  const int Tpad = (T + 31) & ~31;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.y;
  const int i = blockIdx.x * kQB + warp;
  const bool active = i < T;
  const float* kb = kbar + bh * int64_t(T) * D;
  const float* vb = vbar + bh * int64_t(T) * D;
  float* s = srow + warp * Tpad;

  for (int d = lane; d < D; d += 32) qrow[warp * D + d] = active ? qbar[(bh * T + i) * D + d] : 0.f;

  // 1. scores
  for (int j0 = 0; j0 < T; j0 += kKC) {
    __syncthreads();
    const int nj = min(kKC, T - j0);
    for (int x = threadIdx.x; x < nj * D; x += kQB * 32) {
      const int jj = x / D, d = x % D;
      stage[jj * kStride + d] = kb[int64_t(j0 + jj) * D + d];
    }
    __syncthreads();
    if (active && lane < nj) {
      float acc = 0.f;
      const float* kr = stage + lane * kStride;
      const float* qr = qrow + warp * D;
#pragma unroll 16
      for (int d = 0; d < D; ++d) acc = fmaf(qr[d], kr[d], acc);
      s[j0 + lane] = scale * acc;
    }
  }
  __syncwarp();

  // 2. softmax and o_coarse
  float m = -INFINITY;
  for (int j = lane; j < T; j += 32) m = fmaxf(m, s[j]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  float l = 0.f;
  for (int j = lane; j < T; j += 32) l += __expf(s[j] - m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
  float acc[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) acc[c] = 0.f;
  for (int j0 = 0; j0 < T; j0 += kKC) {
    __syncthreads();
    const int nj = min(kKC, T - j0);
    for (int x = threadIdx.x; x < nj * D; x += kQB * 32) {
      const int jj = x / D, d = x % D;
      stage[jj * kStride + d] = vb[int64_t(j0 + jj) * D + d];
    }
    __syncthreads();
    if (active) {
      for (int jj = 0; jj < nj; ++jj) {
        const float p = __expf(s[j0 + jj] - m);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(p, stage[jj * kStride + lane + 32 * c], acc[c]);
      }
    }
  }
  if (!active) return;
  {
    const float inv = 1.0f / l;
    float* oc = o_coarse + (bh * T + i) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) oc[lane + 32 * c] = acc[c] * inv;
  }

  // 3. top-k over video key tiles (video query tiles only)
  if (i < n_p || k <= 0) return;
  const int n_v = T - n_p;
  uint32_t* h = hist + warp * 256;
  uint32_t prefix = 0u, mask = 0u;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int b = 0; b < 8; ++b) h[lane * 8 + b] = 0u;
    __syncwarp();
    for (int j = n_p + lane; j < T; j += 32) {
      const uint32_t key = order_key(s[j]);
      if ((key & mask) == prefix) atomicAdd(h + ((key >> shift) & 255u), 1u);
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
  const uint32_t lt_mask = (1u << lane) - 1u;
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

template <int D>
size_t coarse_smem_bytes(int T) {
  const int Tpad = (T + 31) & ~31;
  return sizeof(float) * (size_t(kKC) * (D + 1) + size_t(kQB) * D + size_t(kQB) * 256 +
                          size_t(kQB) * Tpad);
}

template <int D>
cudaError_t launch_coarse_d(const float* qbar, const float* kbar, const float* vbar, int64_t bh,
                            int T, int n_p, float scale, int k, float* o_coarse, int32_t* topk_idx,
                            float* topk_score, cudaStream_t stream) {
  const size_t smem = coarse_smem_bytes<D>(T);
  cudaError_t e = cudaFuncSetAttribute(coarse_topk_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned((T + kQB - 1) / kQB), unsigned(bh), 1);
  coarse_topk_kernel<D><<<grid, kQB * 32, smem, stream>>>(qbar, kbar, vbar, T, n_p, scale, k,
                                                          o_coarse, topk_idx, topk_score);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_coarse_topk(const float* qbar, const float* kbar, const float* vbar, int64_t bh,
                               int T, int n_p, int D, float scale, int k, float* o_coarse,
                               int32_t* topk_idx, float* topk_score, cudaStream_t stream) {
  if (T > kMaxTiles || bh > 65535) return cudaErrorInvalidValue;
  if (D == 128)
    return launch_coarse_d<128>(qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx,
                                topk_score, stream);
  return launch_coarse_d<64>(qbar, kbar, vbar, bh, T, n_p, scale, k, o_coarse, topk_idx,
                             topk_score, stream);
}

}  // namespace vsa
