// Head projection y = act(x W^T) as a tcgen05 GEMM, written per head: the
// gate's bias-free linear of the layer (SnackOnAI, "The Code, Annotated",
// snippet three: gate = x @ W_gate^T viewed as [.., heads, head_dim]) and,
// with act = identity, any Q/K/V projection of the same shape.
//
//   y[b, h, n, d] = act( sum_c x[b, n, c] * w[h*D + d, c] ),   act = id or sigmoid
//   x bf16 [B, N, C], w bf16 [H*D, C] (nn.Linear layout), y bf16 [B, H, N, D];
//   fp32 accumulation in TMEM, round to nearest even on the store.
//
// Design (one persistent CTA per SM, static round-robin over output tiles of
// 256 rows (tokens) x 256 columns (H*D)).  Tile order: the column tiles are
// split into groups whose W rows take at most 32 MB, and within a group the
// tiles go M-major, so that concurrent CTAs share x rows and one group's W in
// L2 (with all of W, 58 MB at the 42-head gate, W was re-read from DRAM about
// every wave; measured on B200: two groups of 11 and 10 column tiles ran 3-6 %
// faster than one):
//   warp 0  (TMA)       per 64-wide K block, the x box [256 x 64] and the W box
//                       [256 x 64] (128-byte swizzle) into a 3-stage ring.
//   warp 1  (MMA)       one lane issues tcgen05.mma kind::f16, M=128, N=256,
//                       K=16, two per K step (rows 0-127 and 128-255 of the
//                       tile against the same W box), into one TMEM
//                       accumulator of 2 x 256 columns.  A 256 x 256 tile reads
//                       a third fewer operand bytes per FLOP from L2 than
//                       128 x 256 (which bound the earlier kernel), at the
//                       price of a single accumulator.
//   warps 2-9 (epilogue) thread = accumulator row = TMEM lane (warps 2-5 rows
//                       0-127, warps 6-9 rows 128-255): the row's 256 columns
//                       are read with tcgen05.ld in 32-column chunks, passed
//                       through the optional sigmoid and packed to bf16 in
//                       registers; the accumulator is handed back to the MMA
//                       warp before the 16-byte stores into the row's per-head
//                       segments, so the stores overlap the next tile's MMAs.
// Every mbarrier wait is bounded (abort flag + status word, as in the
// attention kernel); rows past B*N and columns past H*D are loaded as zeros by
// TMA and never stored.
#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {
using namespace sm100;

constexpr int kPBM = 256, kPBN = 256, kPBK = 64, kPStages = 3;
constexpr int kPThreads = 320;                  // TMA, MMA, 8 epilogue warps
constexpr int kPABytes = kPBM * kPBK * 2;      // 32 KB
constexpr int kPBBytes = kPBN * kPBK * 2;      // 32 KB
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPHalfA = 128 * kPBK * 2;        // byte offset of rows 128-255 in the x box
constexpr uint32_t kPIdesc = idesc_bf16(128, kPBN, false, false);
// barriers: full[S], empty[S], acc_full, acc_empty, drain
constexpr int kPNBar = 2 * kPStages + 3;
constexpr size_t kPSmem = size_t(kPStages) * kPStageBytes + kPNBar * 8 + 16 + 1024;

struct ProjArgs {
  uint16_t* y;
  unsigned int* status;
  int64_t M;            // B * N rows
  int64_t N;            // tokens per batch element
  int H, D, C;
  int m_tiles, n_tiles, k_blocks;
  int group;            // column tiles per group of the tile order
  int act;              // 0 identity, 1 sigmoid
};

// Tile t -> (row tile m, column tile n): group g holds column tiles
// [g*G, g*G + G) (the last one may be narrower), its tiles in M-major order.
__device__ __forceinline__ void decode_tile(int t, const ProjArgs& a, int& m, int& n) {
  const int G = a.group;
  const int g = t / (a.m_tiles * G), r = t % (a.m_tiles * G);
  const int gw = min(G, a.n_tiles - g * G);
  m = r / gw;
  n = g * G + r % gw;
}

__device__ __forceinline__ float sigmoid_tanh(float g) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * g));
  return fmaf(0.5f, t, 0.5f);
}

__global__ void __launch_bounds__(kPThreads, 1)
    project_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t bar0 = s_base + kPStages * kPStageBytes;
  // full/empty complete once per K block, acc_full/acc_empty once per use of
  // the accumulator; each waiter observes every phase in order
  const uint32_t full = bar0, empty = full + 8 * kPStages, acc_full = empty + 8 * kPStages,
                 acc_empty = acc_full + 8, drain = acc_empty + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kPStages * kPStageBytes + kPNBar * 8);
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + kPStages * kPStageBytes + kPNBar * 8 + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = a.m_tiles * a.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int m, n;
        decode_tile(t, a, m, n);
        for (int kb = 0; kb < a.k_blocks; ++kb, ++g) {
          const uint32_t s = g % kPStages;
          if (g >= uint32_t(kPStages) &&
              !wait_bar(empty + 8 * s, ((g / kPStages) - 1) & 1, abort_flag, a.status, 21)) {
            ok = false;
            break;
          }
          const uint32_t sa = s_base + s * kPStageBytes;
          mbar_expect_tx(full + 8 * s, kPStageBytes);
          tma_load_2d(sa, &tm_x, full + 8 * s, kb * kPBK, m * kPBM);
          tma_load_2d(sa + kPABytes, &tm_w, full + 8 * s, kb * kPBK, n * kPBN);
        }
      }
      if (!ok) {
        // abort: none of our TMA writes may still be in flight
        for (uint32_t x = (g > uint32_t(kPStages) ? g - kPStages : 0); x < g; ++x)
          wait_bar_drain(full + 8 * (x % kPStages), (x / kPStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t g = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
        // the accumulator of the previous tile has been read out
        if (lt >= 1 && !wait_bar(acc_empty, (lt - 1) & 1, abort_flag, a.status, 22)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < a.k_blocks && ok; ++kb, ++g) {
          const uint32_t s = g % kPStages;
          if (!wait_bar(full + 8 * s, (g / kPStages) & 1, abort_flag, a.status, 23)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = s_base + s * kPStageBytes;
#pragma unroll
          for (int ks = 0; ks < kPBK / 16; ++ks) {
            const uint64_t bd = sdesc_sw128(sa + kPABytes + ks * 32, 16, 1024);
            const uint32_t accum = (kb > 0 || ks > 0) ? 1u : 0u;
            umma_bf16(tmem, sdesc_sw128(sa + ks * 32, 16, 1024), bd, kPIdesc, accum);
            umma_bf16(tmem + kPBN, sdesc_sw128(sa + kPHalfA + ks * 32, 16, 1024), bd, kPIdesc,
                      accum);
          }
          umma_commit(empty + 8 * s);
        }
        if (ok) umma_commit(acc_full);
      }
      // drain: every MMA issued above complete before TMEM is freed
      umma_commit(drain);
      wait_bar_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;                       // TMEM lane quadrant of this warp
    const int half = (warp - 2) >> 2;                // rows 0-127 or 128-255 of the tile
    const int row = half * 128 + quad * 32 + lane;
    const uint32_t t_row = tmem + (uint32_t(quad * 32) << 16) + uint32_t(half * kPBN);
    int lt = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
      int m, n;
        decode_tile(t, a, m, n);
      if (!__all_sync(0xFFFFFFFFu, wait_bar(acc_full, lt & 1, abort_flag, a.status, 24))) break;
      tc_fence_after();
      // the row's 256 columns, packed to bf16 pairs in registers
      uint32_t pk[kPBN / 2];
#pragma unroll
      for (int c = 0; c < kPBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_row + 32 * c, v);
        tmem_wait_ld(v);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float lo = __uint_as_float(v[2 * e]), hi = __uint_as_float(v[2 * e + 1]);
          if (a.act == 1) {
            lo = sigmoid_tanh(lo);
            hi = sigmoid_tanh(hi);
          }
          pk[16 * c + e] = pack_bf16(lo, hi);
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);                        // the MMAs of the next tile may start
      const int64_t r = int64_t(m) * kPBM + row;     // global row = b * N + token
      if (r < a.M) {
        const int64_t b = r / a.N, tok = r % a.N;
#pragma unroll
        for (int c = 0; c < kPBN / 32; ++c) {
          const int col0 = n * kPBN + 32 * c;          // 32 columns within one head (D >= 64)
          if (col0 >= a.H * a.D) continue;
          const int h = col0 / a.D, d0 = col0 % a.D;
          uint4* dst = reinterpret_cast<uint4*>(a.y + ((b * a.H + h) * a.N + tok) * a.D + d0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pk[16 * c + 4 * q], pk[16 * c + 4 * q + 1], pk[16 * c + 4 * q + 2],
                                pk[16 * c + 4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u)
                 : "memory");
  }
}

}  // namespace

vsa_status launch_project(const vsa_plan_s* p, const void* x, const void* w, int B, int H, int D,
                          int C, int act, int tiled, void* y, cudaStream_t stream) {
  const int64_t rows_per_b = tiled ? p->n_padded : p->n_tokens;
  const int64_t M = int64_t(B) * rows_per_b;
  const int HD = H * D;
  if (M >= (int64_t(1) << 31) || HD >= (1 << 20))
    return fail(VSA_ERR_UNSUPPORTED, "projection too large for 32-bit TMA coordinates");
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, M, C, kPBM) || !make_map(&mw, w, HD, C, kPBN))
    return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  cudaError_t e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kPSmem));
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, cudaGetErrorString(e));
  ProjArgs a;
  a.y = static_cast<uint16_t*>(y);
  a.status = p->d_status;
  a.M = M;
  a.N = rows_per_b;
  a.H = H;
  a.D = D;
  a.C = C;
  a.m_tiles = int((M + kPBM - 1) / kPBM);
  a.n_tiles = (HD + kPBN - 1) / kPBN;
  a.k_blocks = (C + kPBK - 1) / kPBK;
  {
    // groups of column tiles whose W rows take at most 32 MB
    const int64_t w_bytes = int64_t(HD) * C * 2;
    const int64_t groups = std::max<int64_t>(1, (w_bytes + (int64_t(32) << 20) - 1) >> 25);
    a.group = int((a.n_tiles + groups - 1) / groups);
  }
  a.act = act;
  const int64_t tiles = int64_t(a.m_tiles) * a.n_tiles;
  if (tiles >= (int64_t(1) << 31)) return fail(VSA_ERR_UNSUPPORTED, "too many projection tiles");
  const int grid = int(std::min<int64_t>(tiles, p->num_sms > 0 ? p->num_sms : 148));
  project_kernel<<<grid, kPThreads, kPSmem, stream>>>(mx, mw, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, std::string("projection launch: ") + cudaGetErrorString(e));
  return VSA_OK;
}

}  // namespace vsa
