// HBM-bound passes of the layer: row gather (permute / unpermute), per-tile
// mean pooling, the two fused (permute + pool), and the gated combine.
//
// All three move whole rows of D bf16 values (128 or 256 bytes) as 16-byte
// vectors.  A thread owns one 16-byte chunk of a row per step and keeps
// kUnroll independent loads in flight; consecutive threads walk consecutive
// chunks of the destination, so stores are fully coalesced and every source
// row is read as whole 32-byte sectors.  Grids are sized to a multiple of the
// SM count (8 CTAs of 256 threads per SM) and stride over the work.
#include <cuda_bf16.h>

#include "vsa_internal.h"

namespace vsa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ldg_nc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// dst[bh, r, :] = map[r] >= 0 ? src[bh, map[r], :] : 0.
// kCpr = 16-byte chunks per row (D / 8).
template <int kCpr>
__global__ void __launch_bounds__(kThreads) gather_rows_kernel(const uint4* __restrict__ src,
                                                               uint4* __restrict__ dst,
                                                               const int32_t* __restrict__ map,
                                                               int64_t src_rows, int64_t dst_rows) {
  const int64_t bh = blockIdx.y;
  const uint4* s = src + bh * src_rows * kCpr;
  uint4* d = dst + bh * dst_rows * kCpr;
  const int64_t total = dst_rows * kCpr;
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t c0 = int64_t(blockIdx.x) * kThreads + threadIdx.x; c0 < total;
       c0 += stride * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = c0 + u * stride;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (c < total) {
        const int32_t m = __ldg(map + c / kCpr);
        if (m >= 0) v[u] = ldg_nc(s + int64_t(m) * kCpr + (c % kCpr));
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = c0 + u * stride;
      if (c < total) d[c] = v[u];
    }
  }
}

// Rows of any width (C bf16, C a multiple of 8): dst[b, r, :] = map[r] >= 0 ?
// src[b, map[r], :] : 0.  One warp per destination row; the lanes walk its
// 16-byte chunks with kUnroll loads in flight.  Used to put the layer input
// into tile order before its projections.
__global__ void __launch_bounds__(kThreads) gather_wide_kernel(const uint4* __restrict__ src,
                                                               uint4* __restrict__ dst,
                                                               const int32_t* __restrict__ map,
                                                               int64_t src_rows, int64_t dst_rows,
                                                               int64_t n_rows, int cpr) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (kThreads / 32);
  for (int64_t w = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); w < n_rows;
       w += warps) {
    const int64_t b = w / dst_rows, r = w % dst_rows;
    const int32_t m = __ldg(map + r);
    uint4* d = dst + w * cpr;
    const uint4* s = src + (b * src_rows + (m >= 0 ? m : 0)) * cpr;
    for (int c0 = lane; c0 < cpr; c0 += 32 * kUnroll) {
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = c0 + 32 * u;
        v[u] = (m >= 0 && c < cpr) ? ldg_nc(s + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = c0 + 32 * u;
        if (c < cpr) d[c] = v[u];
      }
    }
  }
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Mean over the live rows of every tile, fp32.  One warp per (tensor, bh, tile):
// 32 / kCpr rows per pass, each lane accumulating 8 columns; lanes that share a
// column group are then summed with shuffles.
template <int kCpr>
__global__ void __launch_bounds__(kThreads) pool_kernel(const uint4* __restrict__ q,
                                                        const uint4* __restrict__ k,
                                                        const uint4* __restrict__ v,
                                                        const int32_t* __restrict__ block_len,
                                                        float* __restrict__ qbar,
                                                        float* __restrict__ kbar,
                                                        float* __restrict__ vbar, int64_t n_items,
                                                        int T, int R) {
  constexpr int kRowsPerPass = 32 / kCpr;
  const int lane = threadIdx.x & 31;
  const int which = blockIdx.y;
  const uint4* src = which == 0 ? q : (which == 1 ? k : v);
  float* out = which == 0 ? qbar : (which == 1 ? kbar : vbar);
  const int64_t warps = int64_t(gridDim.x) * (kThreads / 32);
  for (int64_t item = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); item < n_items;
       item += warps) {
    const int64_t bh = item / T;
    const int t = int(item % T);
    const int n = __ldg(block_len + t);
    const uint4* base = src + ((bh * T + t) * int64_t(R)) * kCpr + (lane % kCpr);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int r = lane / kCpr;
    for (; r + 7 * kRowsPerPass < n; r += 8 * kRowsPerPass) {
      uint4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = ldg_nc(base + int64_t(r + u * kRowsPerPass) * kCpr);
#pragma unroll
      for (int u = 0; u < 8; ++u) add_bf16x8(acc, x[u]);
    }
    for (; r < n; r += kRowsPerPass) add_bf16x8(acc, ldg_nc(base + int64_t(r) * kCpr));
#pragma unroll
    for (int off = kCpr; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
    if (lane < kCpr) {
      const float inv = 1.0f / float(n);
      float4* o = reinterpret_cast<float4*>(out + (bh * T + t) * int64_t(kCpr * 8) + lane * 8);
      o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    }
  }
}

// Permute and pool in one pass (the permute's gather, with the tile mean
// taken on the way): one warp per (bh, tile).  Lane l owns 16-byte chunk
// l % kCpr of rows l / kCpr, l / kCpr + 32 / kCpr, ...; it gathers the tile's
// live rows from their natural positions (row_src), writes the tile's R rows
// contiguously to the permuted layout (zeros past block_len) and adds the
// live rows into 8 fp32 column sums, kU loads in flight.  The lanes that
// share a chunk are then summed with shuffles and the mean written fp32.
// Same HBM bytes as the permute alone; the pooled means cost no extra pass.
template <int kCpr>
__global__ void __launch_bounds__(kThreads) permute_pool_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ row_src,
    const int32_t* __restrict__ block_len, float* __restrict__ pooled, int64_t n_items, int T,
    int R, int64_t src_rows, int64_t dst_rows) {
  constexpr int kRowsPerPass = 32 / kCpr;
  constexpr int kU = 8;
  const int lane = threadIdx.x & 31;
  const int cc = lane % kCpr;
  const int64_t warps = int64_t(gridDim.x) * (kThreads / 32);
  for (int64_t item = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); item < n_items;
       item += warps) {
    const int64_t bh = item / T;
    const int t = int(item % T);
    const int n = __ldg(block_len + t);
    const uint4* s = src + bh * src_rows * kCpr + cc;
    uint4* d = dst + (bh * dst_rows + int64_t(t) * R) * kCpr + cc;
    const int32_t* rs = row_src + int64_t(t) * R;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int r = lane / kCpr; r < R; r += kRowsPerPass * kU) {
      uint4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int rr = r + u * kRowsPerPass;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (rr < n) {
          const int32_t m = __ldg(rs + rr);
          if (m >= 0) v[u] = ldg_nc(s + int64_t(m) * kCpr);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int rr = r + u * kRowsPerPass;
        if (rr < R) {
          d[int64_t(rr) * kCpr] = v[u];
          if (rr < n) add_bf16x8(acc, v[u]);
        }
      }
    }
#pragma unroll
    for (int off = kCpr; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
    if (lane < kCpr) {
      const float inv = 1.0f / float(n);
      float4* o = reinterpret_cast<float4*>(pooled + item * int64_t(kCpr * 8) + lane * 8);
      o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    }
  }
}

// sigmoid(g) = (1 + tanh(g/2)) / 2: one hardware tanh instead of exp + reciprocal.
__device__ __forceinline__ float sigmoidf_(float g) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * g));
  return fmaf(0.5f, t, 0.5f);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// out = o_fine + sigmoid(g) * o_coarse[tile].  The walk is over the padded
// (tiled) rows, so o_fine and g are read contiguously; with kNatural the live
// row r is written to natural token row_src[r] (whole 16-byte chunks of a
// 128/256-byte row), otherwise to row r with pad rows set to 0.
template <int kCpr, bool kNatural>
__global__ void __launch_bounds__(kThreads) gate_combine_kernel(
    const uint4* __restrict__ o_fine, const uint4* __restrict__ gate,
    const float* __restrict__ o_coarse, uint4* __restrict__ out, const int32_t* __restrict__ row_src,
    int64_t n_tokens, int64_t n_padded, int R, int T) {
  const int64_t bh = blockIdx.y;
  const uint4* of = o_fine + bh * n_padded * kCpr;
  const uint4* gg = gate + bh * n_padded * kCpr;
  const float* oc = o_coarse + bh * int64_t(T) * (kCpr * 8);
  uint4* d = out + bh * (kNatural ? n_tokens : n_padded) * kCpr;
  const int64_t total = n_padded * kCpr;
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  constexpr int kU = 2 * kUnroll;
  for (int64_t c0 = int64_t(blockIdx.x) * kThreads + threadIdx.x; c0 < total; c0 += stride * kU) {
    // The data loads do not wait for row_src (pad rows are readable memory),
    // so every load of the step is in flight at once.
    uint4 a[kU], g[kU];
    int32_t src[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t c = c0 + u * stride;
      src[u] = -2;
      if (c < total) {
        src[u] = __ldg(row_src + c / kCpr);
        a[u] = ldg_nc(of + c);
        g[u] = ldg_nc(gg + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t c = c0 + u * stride;
      if (src[u] == -2) continue;                 // past the end
      const int64_t r = c / kCpr;
      const int col = int(c % kCpr);
      uint4 res = make_uint4(0u, 0u, 0u, 0u);
      if (src[u] >= 0) {
        const float4* cp = reinterpret_cast<const float4*>(oc + (r / R) * (kCpr * 8) + col * 8);
        const float4 c0v = __ldg(cp), c1v = __ldg(cp + 1);
        const float cv[8] = {c0v.x, c0v.y, c0v.z, c0v.w, c1v.x, c1v.y, c1v.z, c1v.w};
        const uint32_t aw[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
        const uint32_t gw[4] = {g[u].x, g[u].y, g[u].z, g[u].w};
        uint32_t ow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float f0 = __uint_as_float(aw[i] << 16), f1 = __uint_as_float(aw[i] & 0xFFFF0000u);
          const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
          ow[i] = pack_bf16x2(fmaf(sigmoidf_(g0), cv[2 * i], f0), fmaf(sigmoidf_(g1), cv[2 * i + 1], f1));
        }
        res = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      } else if (kNatural) {
        continue;                                  // pad rows have no natural token
      }
      if (kNatural)
        d[int64_t(src[u]) * kCpr + col] = res;
      else
        d[c] = res;
    }
  }
}

dim3 stream_grid(int num_sms, int64_t bh) {
  const int64_t want = int64_t(num_sms > 0 ? num_sms : 148) * 8;
  int64_t x = (want + bh - 1) / bh;
  if (x < 1) x = 1;
  return dim3(unsigned(x), unsigned(bh), 1);
}

}  // namespace

cudaError_t launch_gather_rows(const uint16_t* src, uint16_t* dst, const int32_t* map, int64_t bh,
                               int64_t src_rows, int64_t dst_rows, int D, int num_sms,
                               cudaStream_t stream) {
  if (bh > 65535) return cudaErrorInvalidValue;
  const dim3 grid = stream_grid(num_sms, bh);
  if (D == 128)
    gather_rows_kernel<16><<<grid, kThreads, 0, stream>>>(reinterpret_cast<const uint4*>(src),
                                                          reinterpret_cast<uint4*>(dst), map,
                                                          src_rows, dst_rows);
  else
    gather_rows_kernel<8><<<grid, kThreads, 0, stream>>>(reinterpret_cast<const uint4*>(src),
                                                         reinterpret_cast<uint4*>(dst), map,
                                                         src_rows, dst_rows);
  return cudaGetLastError();
}

cudaError_t launch_gather_wide(const uint16_t* src, uint16_t* dst, const int32_t* map, int64_t B,
                               int64_t src_rows, int64_t dst_rows, int C, int num_sms,
                               cudaStream_t stream) {
  const int64_t n_rows = B * dst_rows;
  if (n_rows == 0) return cudaSuccess;
  const int64_t want = int64_t(num_sms > 0 ? num_sms : 148) * 8;
  int64_t blocks = (n_rows + 7) / 8;
  if (blocks > want) blocks = want;
  gather_wide_kernel<<<unsigned(blocks), kThreads, 0, stream>>>(
      reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), map, src_rows, dst_rows,
      n_rows, C / 8);
  return cudaGetLastError();
}

cudaError_t launch_pool(const uint16_t* q_t, const uint16_t* k_t, const uint16_t* v_t,
                        const int32_t* block_len, float* qbar, float* kbar, float* vbar,
                        int64_t bh, int T, int R, int D, int num_sms, cudaStream_t stream) {
  const int64_t n_items = bh * T;
  const int64_t want = int64_t(num_sms > 0 ? num_sms : 148) * 8;
  int64_t blocks = (n_items + 7) / 8;
  if (blocks > want) blocks = want;
  const dim3 grid(unsigned(blocks), 3, 1);
  if (D == 128)
    pool_kernel<16><<<grid, kThreads, 0, stream>>>(
        reinterpret_cast<const uint4*>(q_t), reinterpret_cast<const uint4*>(k_t),
        reinterpret_cast<const uint4*>(v_t), block_len, qbar, kbar, vbar, n_items, T, R);
  else
    pool_kernel<8><<<grid, kThreads, 0, stream>>>(
        reinterpret_cast<const uint4*>(q_t), reinterpret_cast<const uint4*>(k_t),
        reinterpret_cast<const uint4*>(v_t), block_len, qbar, kbar, vbar, n_items, T, R);
  return cudaGetLastError();
}

cudaError_t launch_permute_pool(const uint16_t* src, uint16_t* dst, const int32_t* row_src,
                                const int32_t* block_len, float* pooled, int64_t bh, int T, int R,
                                int64_t src_rows, int64_t dst_rows, int D, int num_sms,
                                cudaStream_t stream) {
  const int64_t n_items = bh * T;
  const int64_t want = int64_t(num_sms > 0 ? num_sms : 148) * 8;
  int64_t blocks = (n_items + 7) / 8;
  if (blocks > want) blocks = want;
  if (D == 128)
    permute_pool_kernel<16><<<unsigned(blocks), kThreads, 0, stream>>>(
        reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), row_src, block_len,
        pooled, n_items, T, R, src_rows, dst_rows);
  else
    permute_pool_kernel<8><<<unsigned(blocks), kThreads, 0, stream>>>(
        reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), row_src, block_len,
        pooled, n_items, T, R, src_rows, dst_rows);
  return cudaGetLastError();
}

cudaError_t launch_gate_combine(const uint16_t* o_fine_t, const uint16_t* gate_t,
                                const float* o_coarse, uint16_t* out, int out_natural,
                                const int32_t* row_src, const int32_t* untile, int64_t bh,
                                int64_t n_tokens, int64_t n_padded, int R, int T, int D,
                                int num_sms, cudaStream_t stream) {
  if (bh > 65535) return cudaErrorInvalidValue;
  const dim3 grid = stream_grid(num_sms, bh);
  const uint4* of = reinterpret_cast<const uint4*>(o_fine_t);
  const uint4* g = reinterpret_cast<const uint4*>(gate_t);
  uint4* o = reinterpret_cast<uint4*>(out);
  (void)untile;
  if (D == 128) {
    if (out_natural)
      gate_combine_kernel<16, true><<<grid, kThreads, 0, stream>>>(of, g, o_coarse, o, row_src,
                                                                   n_tokens, n_padded, R, T);
    else
      gate_combine_kernel<16, false><<<grid, kThreads, 0, stream>>>(of, g, o_coarse, o, row_src,
                                                                    n_tokens, n_padded, R, T);
  } else {
    if (out_natural)
      gate_combine_kernel<8, true><<<grid, kThreads, 0, stream>>>(of, g, o_coarse, o, row_src,
                                                                  n_tokens, n_padded, R, T);
    else
      gate_combine_kernel<8, false><<<grid, kThreads, 0, stream>>>(of, g, o_coarse, o, row_src,
                                                                   n_tokens, n_padded, R, T);
  }
  return cudaGetLastError();
}

}  // namespace vsa
