// Block-sparse fine attention over the kept K/V tiles (step 4 of the layer),
// for sm_100a: TMA tile loads driven by the kept-tile list, tcgen05 MMAs that
// accumulate in tensor memory (TMEM), and an online softmax.
//
// Semantics (SnackOnAI, "The Code, Annotated", snippet two: sink_blocks and
// sink_q = [0, num_prefix_tiles), block_len): query tile i attends to every
// tile when i < n_p (prefix queries are dense) and to the n_p prefix sink tiles
// plus its kept video tiles otherwise; key rows at or past block_len[j] are
// masked; o = softmax(scale * q k^T) v per live query row.
//
// Design (one persistent CTA per SM; work items handed out in order from a
// per-plan global counter):
//   work item = (b*h, query tile i); the video items come first, head by
//   head, and the prefix items (n_p per head, each T key tiles long,
//   streaming a whole head's K/V) come last.  The TMA K warp takes the next
//   item from the counter (atomicAdd) and publishes it to the other roles
//   through one of two shared-memory slots.  Taken in order, the items in
//   flight span one or two heads, whose K/V stay in L2; a static split let
//   CTAs drift apart by several heads, and prefix items run first kept their
//   CTAs a millisecond behind for the rest of the launch.
//   warp 8  (TMA K)  loads Q once per item (evict-first: it is read once) and
//                    K_j per kept tile into a K ring.
//   warp 9  (TMA V)  loads V_j into its own ring (V is needed later than K).
//   warp 10 (MMA S)  one lane issues S_n = Q K_n^T (M=128, N=R, K=D) into the
//                    TMEM S tile of softmax warpgroup n & 1 once that warpgroup
//                    has read its previous S.
//   warp 11 (MMA PV) one lane issues O += P_n V_n (M=128, N=D, K=R) with the A
//                    operand P_n read from TMEM; the two issuers run
//                    independently (S and PV touch disjoint TMEM columns).
//   warps 0-7        two softmax warpgroups; warpgroup w takes the tiles
//                    n = w (mod 2) of an item (a split of the key set inside the
//                    CTA), and both add into one O.  Thread = query row = TMEM
//                    lane: it loads its S row, masks past block_len, and scales
//                    by a reference max m_ref shared by both warpgroups.  m_ref
//                    after tile n is decided by the warp that runs tile n, from
//                    m_ref after tile n-1 (published by the warp of the other
//                    warpgroup on the same TMEM lanes through a shared-memory
//                    mailbox) and its own row max; it moves only when a row grew
//                    by more than 2^8 (exact: p <= 256), and then that warp
//                    rescales its O rows once PV_{n-1} is complete.  P = exp2(.)
//                    goes to TMEM as bf16 pairs.  The epilogue adds the two
//                    warpgroups' row sums and stores bf16 rows (and the LSE), or
//                    the gated combine in natural order.
// TMEM columns: O [0,D), S_w [D + w*128, D + (w+1)*128), P_w [D + 256 + w*64,
// D + 256 + (w+1)*64) (two bf16 per 32-bit column, key order, row = lane).
// S_{n+2} depends only on S_n having been read, P_n only on PV_{n-2}, so MMA
// latency stays off the softmax's path, and no P tile takes shared memory.
//
// 64-row tiles (VSA 4x4x4 cubes) run in pairs, so that every MMA keeps its
// 128 x 128 shape: an item is a pair of consecutive query tiles (2m, 2m+1) of
// one head (MMA rows 0-63 and 64-127; their 128 rows are contiguous in the
// tiled layout, so one Q box loads both), and a step is a pair of key tiles
// taken in ascending order from the union of the two query tiles' key sets.
// Each entry of that list carries a mask of the query tiles whose set holds
// it; the softmax warps of the other query tile set its scores to -inf in
// registers, so that both query tiles run one branch-free path (row max,
// exponentials, P) in which those keys count for nothing (measured on B200: 6 %
// faster than skipping their exponentials on a separate path, whose code the
// two halves of a pair then ran at once).  A key tile both query tiles kept is
// loaded once for both.
// The list is built per item by the K producer warp (two bitmaps over the T
// tiles, then a ballot compaction) into one of two shared-memory slots that
// the other roles read.
//
// Every mbarrier wait is bounded (kWaitLimitNs of wall time); on expiry the
// CTA raises an abort flag, records VSA_ERR_DEVICE_TIMEOUT in the status word,
// drains its own TMA loads and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {
using namespace sm100;

constexpr int kBM = 128;                 // MMA M (query rows per item)
constexpr int kThreadsAttn = 384;        // 8 softmax warps + TMA K + TMA V + MMA S + MMA PV
constexpr int kWarpTmaK = 8, kWarpTmaV = 9, kWarpMmaS = 10, kWarpMmaPV = 11;

// K and V ring depths for 128-row tiles (tuning knobs, bounded by shared memory).
#ifndef VSA_NSK128
#define VSA_NSK128 3
#endif
#ifndef VSA_NSV128
#define VSA_NSV128 2
#endif

// Tuning knobs (compile-time).  L2 prefetch distance of the K producer in
// key tiles (0: none), work item order (see decode_item), an evict-first L2
// policy on the Q loads (each Q tile is read once) and an evict-last policy
// on the K/V loads (each K/V tile is read by many query tiles).  Measured on
// B200 at the 104k-token Veda layer (sparse attention + combine): item order
// 0 -> 1 took 27.0 to 25.6 ms; a 4-tile L2 prefetch cost 0.5-0.9 ms (it
// doubles the L2 lookups, and the co-resident CTAs already share most K/V
// tiles); the K/V evict-last policy and streaming epilogue accesses changed
// nothing measurable or cost a little.
#ifndef VSA_PREFETCH
#define VSA_PREFETCH 0
#endif
#ifndef VSA_ORDER
#define VSA_ORDER 1
#endif
#ifndef VSA_QHINT
#define VSA_QHINT 1
#endif
#ifndef VSA_KVHINT
#define VSA_KVHINT 0
#endif
// Streaming (evict-first) gate loads and output stores in the fused epilogue.
#ifndef VSA_STREAM_IO
#define VSA_STREAM_IO 0
#endif
constexpr int kItemOrder = VSA_ORDER;

// Progress trace for debugging builds (-DVSA_TRACE): each role of each CTA
// publishes its position in the pipeline to a host-visible buffer (16 slots
// per CTA).  Compiled out otherwise.
#ifdef VSA_TRACE
__device__ unsigned int* vsa_trace_buf = nullptr;
__device__ __forceinline__ void vsa_trace(int slot, unsigned int v) {
  if (vsa_trace_buf != nullptr) {
    reinterpret_cast<volatile unsigned int*>(vsa_trace_buf)[blockIdx.x * 16 + slot] = v;
    __threadfence_system();
  }
}
#define VSA_TR(slot, code, g) vsa_trace((slot), (unsigned(g) << 8) | unsigned(code))
#else
#define VSA_TR(slot, code, g) ((void)0)
#endif

// Event timeline for debugging builds (-DVSA_TIMELINE): CTA 0 records
// (role, event, tile, SM clock) into a device buffer, 4096 entries per role.
#ifdef VSA_TIMELINE
__device__ unsigned long long* vsa_tl_buf = nullptr;
__device__ __forceinline__ void vsa_tl(int role, unsigned int ev, unsigned int tile,
                                       unsigned int& k) {
  if (vsa_tl_buf != nullptr && blockIdx.x == 0) {
    if (k < 4096u) {
      long long c;
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(c));
      vsa_tl_buf[role * 4096 + k] = (unsigned long long)(c & 0xFFFFFFFFFFull) |
                                    ((unsigned long long)(ev & 0xFFu) << 40) |
                                    ((unsigned long long)(tile & 0xFFFFu) << 48);
      ++k;
    }
  }
}
#define VSA_TL(role, ev, tile) vsa_tl((role), (ev), (tile), tl_k)
#define VSA_TL_DECL unsigned int tl_k = 0
#else
#define VSA_TL(role, ev, tile) ((void)0)
#define VSA_TL_DECL ((void)0)
#endif

// PTX wrappers, bounded waits and the tensor-map encoder: sm100.cuh.

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe, to take part of the exponentials off the MUFU unit.
// Cody-Waite range reduction: j = round(x) through the 1.5*2^23 magic constant
// (the fp32 add rounds to nearest and leaves j in the low mantissa bits), f =
// x - j in [-1/2, 1/2]; 2^f by a degree-3 polynomial fitted to minimise the
// relative error on that interval (max 2.2e-4, far below bf16's 2^-9); 2^j is
// added to the exponent field.  x is clamped at -125 so the exponent stays
// normal (the result is then ~2.4e-38, nothing for any sum it enters).

#ifndef VSA_EXP2_FMA_SHARE
#define VSA_EXP2_FMA_SHARE 0
#endif
// One exponential in kExp2FmaShare runs on the FMA pipe (0: all on MUFU).  On
// B200 every share measured slower (27.6 ms with none, 28.6 / 30.7 / 31.6 ms
// with 1 in 8 / 4 / 2 on an earlier kernel; 24.0 ms with none, 25.6 / 35.4 ms
// with 1 in 16 / 8 on the current one), so it is off.
constexpr int kExp2FmaShare = VSA_EXP2_FMA_SHARE;
// The reference-max decision of a tile is published after this many of the
// tile's 32-score exponential chunks (R/32 or more: after all of them), so
// that the partner warp's exponentials start while ours finish.  Measured on
// B200 (104k-token Veda layer, attention + combine): after all 4 chunks
// 24.5 ms, after 3 23.3 ms, after 2 23.1 ms, after 1 29.2 ms.
#ifndef VSA_PUB_CHUNK
#define VSA_PUB_CHUNK 2
#endif
constexpr int kPubChunk = VSA_PUB_CHUNK;
constexpr float kExp2C0 = 0.99996275f;
constexpr float kExp2C1 = 0.69358679f;
constexpr float kExp2C2 = 0.24215202f;
constexpr float kExp2C3 = 0.05286738f;
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction, two lanes of work).
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---------------------------------------------------------------- kernel

struct AttnArgs {
  const int32_t* topk;        // [BH, n_v, k]
  const int32_t* block_len;   // [T]
  uint16_t* out;              // bf16 [BH, N_pad, D], or [BH, N, D] natural when fused
  float* lse;                 // [BH, N_pad] or null
  unsigned int* status;       // device status word
  unsigned long long wait_ns; // bound of every mbarrier wait (kWaitLimitNs unless shortened)
  unsigned int* work;         // paired tiles: [next item, CTAs done], zero at launch
  // fused gated combine (step 5) in the epilogue: out[row_src[r]] =
  // o_fine[r] + sigmoid(gate[row_src[r]]) * o_coarse[tile(r)]
  const uint16_t* gate;       // bf16 [BH, N, D] natural order, or null (unfused)
  const float* o_coarse;      // fp32 [BH, T, D]
  const int32_t* row_src;     // [N_pad] padded row -> token, -1 for a pad row
  int T, n_p, k, n_items, BH;
  int64_t n_pad, n_tok;
  float scale_log2;           // scale * log2(e)
  // reference thinning: the kept reference tiles of each video query tile
  // [BH, n_v, k_ref], or null (every reference tile is a sink)
  int k_ref;
  int n_sink;                 // reference tiles of a video item: k_ref, or n_p
  const int32_t* topk_ref;
};

// sigmoid(g) = (1 + tanh(g/2)) / 2 with the hardware tanh.
__device__ __forceinline__ float sigmoid_fast(float g) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * g));
  return fmaf(0.5f, t, 0.5f);
}

template <int R, int D>
struct Cfg {
  // 64-row tiles run in pairs: two query tiles per item, two key tiles per step
  static constexpr bool kPair = (R == 64);
  static constexpr int BN = 128;                         // key rows per step
  static constexpr int NSK = VSA_NSK128;                 // K ring stages
  static constexpr int NSV = VSA_NSV128;                 // V ring stages
  static constexpr int QBYTES = kBM * D * 2;
  static constexpr int TBYTES = BN * D * 2;              // one step's K (or V) rows
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + NSK * TBYTES;
  // reference-max mailbox fp32 [2 tile parities][128 rows], then the
  // epilogue's (m, l) exchange fp32 [2 values][2 warpgroups][128 rows]
  static constexpr int OFF_X = OFF_V + NSV * TBYTES;
  static constexpr int OFF_BAR = OFF_X + (2 + 4) * 128 * 4;
  // barriers: q_full, q_empty, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV],
  //           s_full[2], s_empty[2], p_full[2], pv_done[2], dec[4], o_full, o_empty,
  //           drain, drain2, list_full[2], list_empty[2] (paired tiles)
  static constexpr int NBAR = 2 + 2 * NSK + 2 * NSV + 8 + 4 + 4 + 4;
  // barriers, then the tmem slot, the abort flag and (128-row tiles) the
  // item of each of the two list slots
  static constexpr int TAIL = NBAR * 8 + 16;
  // TMEM columns: O [0, D), S_w [D + w*BN, D + (w+1)*BN), P_w (bf16 pairs)
  // [D + 2*BN + w*BN/2, D + 2*BN + (w+1)*BN/2)
  static constexpr uint32_t COL_O = 0;
  static constexpr uint32_t COL_S = D;
  static constexpr uint32_t COL_P = D + 2 * BN;
  static constexpr uint32_t TMEM_COLS = (D + 3 * BN) <= 256 ? 256u : 512u;
  static_assert(D + 3 * BN <= 512, "TMEM columns");
  static constexpr uint32_t IDESC_QK = idesc_bf16(kBM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16(kBM, D, false, true);
  // bytes: tiles, exchanges, barriers/misc, then the lists: blen uint8[T] and
  // two int32[k] kept-tile lists; paired tiles: the two list lengths, two
  // bitmaps of ceil(T/32) words and two list slots of list_cap(T) entries
  __host__ __device__ static int list_cap(int T) { return (T + 3) & ~3; }
  __host__ __device__ static int bitmap_words(int T) { return (T + 31) >> 5; }
  static size_t bytes(int T, int k) {
    if (kPair)
      return size_t(OFF_BAR) + TAIL + 16 + size_t(8) * ((bitmap_words(T) + 3) & ~3) +
             size_t(8) * list_cap(T);
    return size_t(OFF_BAR) + TAIL + size_t((T + 15) & ~15) + size_t(8) * ((k + 3) & ~3);
  }
};

// List entry of the paired kernel: key tile index | mask << 16 (bit h: query
// tile 2m+h holds it) | (block_len - 1) << 18.
constexpr uint32_t kEntryTile = 0xFFFFu;
__device__ __forceinline__ int entry_tile(uint32_t e) { return int(e & kEntryTile); }
__device__ __forceinline__ bool entry_has(uint32_t e, int half) { return (e >> (16 + half)) & 1u; }
__device__ __forceinline__ int entry_blen(uint32_t e) { return int((e >> 18) & 63u) + 1; }

// Pair item -> (b*h, pair m): the pairs made of video tiles only first, head
// by head, then the pairs that hold a prefix tile (dense, T key tiles long),
// as decode_item orders single tiles.
__device__ __forceinline__ void decode_pair(int item, int BH, int n_pp, int n_pairs, int64_t& bh,
                                            int& m) {
  const int nvp = n_pairs - n_pp;
  const int first = BH * nvp;
  if (item < first) {
    bh = item / nvp;
    m = n_pp + item % nvp;
  } else {
    const int v = item - first;
    bh = v / n_pp;
    m = v % n_pp;
  }
}

// Work item -> (b*h, query tile i).  kItemOrder 0: every head's prefix query
// tiles first, then the video query tiles head by head; 1: the video tiles
// head by head, then every head's prefix tiles; 2: head by head, each head's
// tiles in tile order.
__device__ __forceinline__ void decode_item(int item, int BH, int n_p, int n_v, int64_t& bh,
                                            int& i) {
  if (kItemOrder == 2) {
    bh = item / (n_p + n_v);
    i = item % (n_p + n_v);
    return;
  }
  const int first = kItemOrder == 0 ? BH * n_p : BH * n_v;
  const bool prefix = kItemOrder == 0 ? item < first : item >= first;
  const int v = kItemOrder == 0 ? (prefix ? item : item - first) : (prefix ? item - first : item);
  if (prefix) {
    bh = v / n_p;
    i = v % n_p;
  } else {
    bh = v / n_v;
    i = n_p + v % n_v;
  }
}

// Kept video tile x of item (bh, i), clamped into [n_p, T) (recording a fault).
__device__ __forceinline__ int kept_tile(const AttnArgs& a, int64_t bh, int i, int x) {
  const int n_v = a.T - a.n_p;
  int j = __ldg(a.topk + (bh * n_v + (i - a.n_p)) * int64_t(a.k) + x);
  if (j < a.n_p || j >= a.T) {
    record(a.status, kStatusBadIndex, unsigned(j));
    j = a.n_p;
  }
  return j;
}

// Reference key tile x (< n_sink) of video item (bh, i): tile x when every
// reference tile is kept, else the item's x-th kept reference tile, clamped
// into [0, n_p) (recording a fault).
__device__ __forceinline__ int sink_tile(const AttnArgs& a, int64_t bh, int i, int x) {
  if (a.topk_ref == nullptr) return x;
  const int n_v = a.T - a.n_p;
  int j = __ldg(a.topk_ref + (bh * n_v + (i - a.n_p)) * int64_t(a.k_ref) + x);
  if (j < 0 || j >= a.n_p) {
    record(a.status, kStatusBadIndex, unsigned(j));
    j = 0;
  }
  return j;
}

// Reference tiles a video item attends to: all n_p, or the k_ref listed ones
// when the kernel is built for reference thinning (kRef).  A template flag,
// so that the unthinned kernel carries none of the list's arithmetic.
template <bool kRef>
__device__ __forceinline__ int n_sink(const AttnArgs& a) {
  return kRef ? a.n_sink : a.n_p;
}

// Key tile of step x of item (bh, i): every tile in order for a dense
// (prefix) item; else the reference tiles, then the kept video tiles, read
// from the item's shared-memory list (step_tile) or from the kept-tile array
// (step_tile_global).
template <bool kRef>
__device__ __forceinline__ int step_tile(const AttnArgs& a, int64_t bh, int i, bool dense, int x,
                                         const int32_t* list) {
  const int ns = n_sink<kRef>(a);
  if (dense || x < ns) return (kRef && !dense) ? sink_tile(a, bh, i, x) : x;
  return list[x - ns];
}
template <bool kRef>
__device__ __forceinline__ int step_tile_global(const AttnArgs& a, int64_t bh, int i, bool dense,
                                                int x) {
  const int ns = n_sink<kRef>(a);
  if (dense || x < ns) return (kRef && !dense) ? sink_tile(a, bh, i, x) : x;
  return kept_tile(a, bh, i, x - ns);
}

// Producer loop shared by the K and the V warp: lane 0 issues one TMA tile per
// kept key tile into an NS-stage ring; the K warp also loads Q per item and
// (kPrefetch > 0) prefetches K/V tiles kPrefetch ahead into L2.
template <int R, int D, int NS, bool kIsK, bool kRef>
__device__ __forceinline__ void producer(const AttnArgs& a, const CUtensorMap* tm_q,
                                         const CUtensorMap* tm_t, const CUtensorMap* tm_other,
                                         uint32_t sQ, uint32_t sT, uint32_t full, uint32_t empty,
                                         uint32_t q_full, uint32_t q_empty, int32_t* s_list,
                                         uint32_t list_full, uint32_t list_empty, int* items,
                                         volatile int* abort_flag, int lane, int BH, int n_v) {
  using C = Cfg<R, D>;
  constexpr int kPrefetch = VSA_PREFETCH;
  VSA_TL_DECL;
  uint32_t g = 0, q_issued = 0;
  int t = 0;
  bool ok = true;
  for (; ok; ++t) {
    // the item: the K warp takes the next one of the grid (head-major order)
    // from the work counter and publishes it in slot t & 1 (-1: none left)
    const int slot = t & 1;
    int item = 0;
    if (kIsK) {
      if (t >= 2)
        ok = __all_sync(0xFFFFFFFFu, wait_bar(list_empty + 8 * slot, ((t >> 1) - 1) & 1, abort_flag,
                                              a.status, 27, a.wait_ns));
      if (!ok) break;
      if (lane == 0) item = int(atomicAdd(a.work, 1u));
      item = __shfl_sync(0xFFFFFFFFu, item, 0);
      if (lane == 0) {
        items[slot] = item < a.n_items ? item : -1;
        mbar_arrive(list_full + 8 * slot);
      }
      __syncwarp();
      if (item >= a.n_items) break;
    } else {
      ok = __all_sync(0xFFFFFFFFu,
                      wait_bar(list_full + 8 * slot, (t >> 1) & 1, abort_flag, a.status, 28, a.wait_ns));
      if (!ok) break;
      item = items[slot];
      if (item < 0) break;
    }
    int64_t bh;
    int i;
    decode_item(item, BH, a.n_p, n_v, bh, i);
    const bool dense = i < a.n_p;
    const int nk = dense ? a.T : n_sink<kRef>(a) + a.k;
    if (!dense)
      for (int x = lane; x < a.k; x += 32) s_list[x] = kept_tile(a, bh, i, x);
    __syncwarp();
    if (lane == 0) {
      const int64_t row0 = bh * a.n_pad;
      if (kIsK) {
        VSA_TR(8, 1, g);
        if (t > 0) ok = wait_bar(q_empty, (t - 1) & 1, abort_flag, a.status, 1, a.wait_ns);
        if (ok) {
          ++q_issued;
          mbar_expect_tx(q_full, C::QBYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            if (VSA_QHINT)
              tma_load_2d_hint(sQ + c * kBM * 128, tm_q, q_full, c * 64, int(row0 + int64_t(i) * R),
                               l2_evict_first_policy());
            else
              tma_load_2d(sQ + c * kBM * 128, tm_q, q_full, c * 64, int(row0 + int64_t(i) * R));
        }
      }
      for (int n = 0; n < nk && ok; ++n, ++g) {
        const uint32_t s = g % NS;
        VSA_TL(kIsK ? 3 : 4, 'x', g);
        if (g >= uint32_t(NS)) {
          ok = wait_bar(empty + 8 * s, ((g / NS) - 1) & 1, abort_flag, a.status, kIsK ? 2 : 11, a.wait_ns);
          if (!ok) break;
        }
        VSA_TL(kIsK ? 3 : 4, kIsK ? 'K' : 'V', g);
        const int j = step_tile<kRef>(a, bh, i, dense, n, s_list);
        const int row = int(row0 + int64_t(j) * R);
        mbar_expect_tx(full + 8 * s, C::TBYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          if (VSA_KVHINT)
            tma_load_2d_hint(sT + s * C::TBYTES + c * C::BN * 128, tm_t, full + 8 * s, c * 64, row,
                             l2_evict_last_policy());
          else
            tma_load_2d(sT + s * C::TBYTES + c * C::BN * 128, tm_t, full + 8 * s, c * 64, row);
        if (kIsK && kPrefetch > 0 && n + kPrefetch < nk) {
          const int jp = step_tile<kRef>(a, bh, i, dense, n + kPrefetch, s_list);
          const int rp = int(row0 + int64_t(jp) * R);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_prefetch_l2(tm_t, c * 64, rp);
            tma_prefetch_l2(tm_other, c * 64, rp);
          }
        }
        VSA_TR(kIsK ? 8 : 9, 4, g);
      }
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(list_empty + 8 * slot);
  }
  if (lane == 0 && !ok) {
    // Abort: make sure none of our TMA writes is still in flight.
    for (uint32_t x = (g > uint32_t(NS) ? g - NS : 0); x < g; ++x)
      wait_bar_drain(full + 8 * (x % NS), (x / NS) & 1);
    if (kIsK && q_issued > 0) wait_bar_drain(q_full, (q_issued - 1) & 1);
  }
}

// Union key list of pair m of head bh (whole warp): bit j of bitmap h is set
// when query tile 2m+h attends to key tile j (every tile for a dense prefix
// query tile; its reference tiles and kept video tiles otherwise; none when
// 2m+h = T); the list holds every j with a bit set, ascending, as packed
// entries.  Returns its length.  Out-of-range kept indices are clamped and
// recorded as by kept_tile / sink_tile.
template <bool kRef>
__device__ int build_pair_list(const AttnArgs& a, int64_t bh, int m, uint32_t* bm, uint32_t* list,
                               int lane) {
  const int T = a.T, W = (T + 31) >> 5;
  for (int h = 0; h < 2; ++h) {
    const int i = 2 * m + h;
    uint32_t* b = bm + h * W;
    const bool dense = i < a.n_p;
    for (int w = lane; w < W; w += 32) {
      const int rem = T - 32 * w;
      b[w] = !dense ? 0u : (rem >= 32 ? 0xFFFFFFFFu : ((1u << rem) - 1u));
    }
    __syncwarp();
    if (!dense && i < T) {
      const int ns = n_sink<kRef>(a);
      for (int x = lane; x < ns + a.k; x += 32) {
        const int j = x < ns ? (kRef ? sink_tile(a, bh, i, x) : x) : kept_tile(a, bh, i, x - ns);
        atomicOr(b + (j >> 5), 1u << (j & 31));
      }
    }
    __syncwarp();
  }
  int count = 0;
  for (int w = 0; w < W; ++w) {
    const uint32_t w0 = bm[w], w1 = bm[W + w];
    const uint32_t mask = ((w0 >> lane) & 1u) | (((w1 >> lane) & 1u) << 1);
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, mask != 0u);
    if (mask != 0u) {
      const int j = 32 * w + lane;              // < T: no bit past T is ever set
      list[count + __popc(ball & ((1u << lane) - 1u))] =
          uint32_t(j) | (mask << 16) | (uint32_t(__ldg(a.block_len + j) - 1) << 18);
    }
    count += __popc(ball);
  }
  if (lane == 0 && (count & 1)) list[count] = 0u;   // an odd list's last step: no tile b
  __syncwarp();
  return count;
}

// Producers of the paired kernel (64-row tiles).  The K warp builds each
// item's union list into list slot t & 1 (after every reader has released
// the slot's previous item) and publishes it; the V warp waits for it.  Lane
// 0 then loads, per step, key tiles 2n and 2n+1 of the list into one ring slot
// (rows 0-63 and 64-127 of each 64-column box); the second tile of an
// odd-length list's last step is read from the rows before the tensor, which
// load as zeros.  The K warp also loads the item's 128 query rows (tiles 2m,
// 2m+1).  Both release the list slot once their loads are issued.
template <int D, int NS, bool kIsK, bool kRef>
__device__ __forceinline__ void producer_pair(const AttnArgs& a, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_t, uint32_t sQ, uint32_t sT,
                                              uint32_t full, uint32_t empty, uint32_t q_full,
                                              uint32_t q_empty, uint32_t list_full,
                                              uint32_t list_empty, uint32_t* lists, int* counts,
                                              uint32_t* bm, int cap, volatile int* abort_flag,
                                              int lane) {
  using C = Cfg<64, D>;
  const int n_pairs = (a.T + 1) >> 1, n_pp = (a.n_p + 1) >> 1;
  uint32_t g = 0, q_issued = 0;
  int t = 0;
  bool ok = true;
  for (; ok; ++t) {
    int64_t bh;
    int m;
    const int slot = t & 1;
    uint32_t* list = lists + slot * cap;
    int count;
    if (kIsK) {
      if (t >= 2)
        ok = __all_sync(0xFFFFFFFFu, wait_bar(list_empty + 8 * slot, ((t >> 1) - 1) & 1, abort_flag,
                                              a.status, 22, a.wait_ns));
      if (!ok) break;
      // the next item of the whole grid, in the head-major item order
      int item = 0;
      if (lane == 0) item = int(atomicAdd(a.work, 1u));
      item = __shfl_sync(0xFFFFFFFFu, item, 0);
      if (item >= a.n_items) {          // none left: publish the end
        if (lane == 0) {
          counts[slot] = -1;
          mbar_arrive(list_full + 8 * slot);
        }
        __syncwarp();
        break;
      }
      decode_pair(item, a.BH, n_pp, n_pairs, bh, m);
      count = build_pair_list<kRef>(a, bh, m, bm, list, lane);
      if (lane == 0) {
        counts[slot] = count;
        counts[2 + slot] = item;
        mbar_arrive(list_full + 8 * slot);
      }
      __syncwarp();
    } else {
      ok = __all_sync(0xFFFFFFFFu,
                      wait_bar(list_full + 8 * slot, (t >> 1) & 1, abort_flag, a.status, 23, a.wait_ns));
      if (!ok) break;
      count = counts[slot];
      if (count < 0) break;              // no item left
      decode_pair(counts[2 + slot], a.BH, n_pp, n_pairs, bh, m);
    }
    const int nk = (count + 1) >> 1;
    if (lane == 0) {
      const int64_t row0 = bh * a.n_pad;
      if (kIsK) {
        if (t > 0) ok = wait_bar(q_empty, (t - 1) & 1, abort_flag, a.status, 1, a.wait_ns);
        if (ok) {
          ++q_issued;
          mbar_expect_tx(q_full, C::QBYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d_hint(sQ + c * kBM * 128, tm_q, q_full, c * 64, int(row0 + int64_t(m) * 128),
                             l2_evict_first_policy());
        }
      }
      for (int n = 0; n < nk && ok; ++n, ++g) {
        const uint32_t s = g % NS;
        if (g >= uint32_t(NS)) {
          ok = wait_bar(empty + 8 * s, ((g / NS) - 1) & 1, abort_flag, a.status, kIsK ? 2 : 11, a.wait_ns);
          if (!ok) break;
        }
        const int row_a = int(row0 + int64_t(entry_tile(list[2 * n])) * 64);
        const int row_b =
            2 * n + 1 < count ? int(row0 + int64_t(entry_tile(list[2 * n + 1])) * 64) : -64;
        mbar_expect_tx(full + 8 * s, C::TBYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const uint32_t dst = sT + s * C::TBYTES + c * C::BN * 128;
          tma_load_2d(dst, tm_t, full + 8 * s, c * 64, row_a);
          tma_load_2d(dst + 64 * 128, tm_t, full + 8 * s, c * 64, row_b);
        }
      }
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(list_empty + 8 * slot);
  }
  if (lane == 0 && !ok) {
    // Abort: make sure none of our TMA writes is still in flight.
    for (uint32_t x = (g > uint32_t(NS) ? g - NS : 0); x < g; ++x)
      wait_bar_drain(full + 8 * (x % NS), (x / NS) & 1);
    if (kIsK && q_issued > 0) wait_bar_drain(q_full, (q_issued - 1) & 1);
  }
}

// Score columns of the key rows past block_len of a partial 64-row key tile
// (tile a: columns [0, 64), tile b: [64, 128) of the S row at taddr) set to
// -inf in TMEM, so that the row max and the exponentials need no mask.  A
// call, not inline code: partial tiles are rare and the softmax's common
// path stays as compact as it is without them.  Whole warp, warp-uniform
// arguments.
__device__ __noinline__ void mask_partial_tiles(uint32_t taddr, int bla, int blb) {
  const uint32_t ninf = __float_as_uint(-INFINITY);
  if (bla > 0)
    for (int col = bla; col < 64; ++col) tmem_st1(taddr + col, ninf);
  if (blb > 0)
    for (int col = blb; col < 64; ++col) tmem_st1(taddr + 64 + col, ninf);
  tmem_wait_st();
}
// The same for one 128-row key tile: columns [bl, 128) of the S row.
__device__ __noinline__ void mask_tile_tail(uint32_t taddr, int bl) {
  const uint32_t ninf = __float_as_uint(-INFINITY);
  for (int col = bl; col < 128; ++col) tmem_st1(taddr + col, ninf);
  tmem_wait_st();
}

template <int R, int D, bool kRef>
__global__ void __launch_bounds__(kThreadsAttn, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = Cfg<R, D>;
  constexpr int BN = C::BN, NSK = C::NSK, NSV = C::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t sQ = s_base + C::OFF_Q, sK = s_base + C::OFF_K, sV = s_base + C::OFF_V;
  const uint32_t bar0 = s_base + C::OFF_BAR;
  const uint32_t q_full = bar0, q_empty = bar0 + 8;
  const uint32_t k_full = bar0 + 16, k_empty = k_full + 8 * NSK;
  const uint32_t v_full = k_empty + 8 * NSK, v_empty = v_full + 8 * NSV;
  // s_full[w], s_empty[w], p_full[w] and pv_done[w] complete once per tile of
  // warpgroup w, dec[q] once per tile (the reference-max decision for TMEM
  // lane quadrant q), o_full and o_empty once per item.  Every wait targets a
  // phase whose predecessor is already complete and whose successor cannot
  // complete before the waiter has observed it, so the parity test never
  // aliases.
  // Paired tiles: list_full[slot] completes once per item that uses the list
  // slot (the K warp published its list), list_empty[slot] once every reader
  // has released it (K and V warps, the two issuers, the eight softmax warps).
  const uint32_t s_full = v_empty + 8 * NSV, s_empty = s_full + 16, p_full = s_empty + 16,
                 pv_done = p_full + 16, dec = pv_done + 16, o_full = dec + 32,
                 o_empty = o_full + 8, drain = o_empty + 8, drain2 = drain + 8,
                 list_full = drain2 + 8, list_empty = list_full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + C::NBAR * 8 + 4);
  float* mbox = reinterpret_cast<float*>(smem + C::OFF_X);       // [2][128]
  float* x_m = mbox + 2 * 128;                                    // [2][128]
  float* x_l = x_m + 2 * 128;                                     // [2][128]
  uint8_t* s_blen = smem + C::OFF_BAR + C::TAIL;                  // [T]
  int32_t* s_klist = reinterpret_cast<int32_t*>(s_blen + ((a.T + 15) & ~15));
  int32_t* s_vlist = s_klist + ((a.k + 3) & ~3);
  // 128-row tiles: the item of each list slot (-1: none left)
  int* r_items = reinterpret_cast<int*>(smem + C::OFF_BAR + C::NBAR * 8 + 8);
  // paired tiles: list lengths [2], bitmaps [2][W], list slots [2][cap]
  int* p_counts = reinterpret_cast<int*>(smem + C::OFF_BAR + C::TAIL);
  uint32_t* p_bm = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::TAIL + 16);
  const int p_cap = C::list_cap(a.T);
  uint32_t* p_lists = p_bm + 2 * ((C::bitmap_words(a.T) + 3) & ~3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_v = a.T - a.n_p;
  const int BH = a.n_items / (C::kPair ? (a.T + 1) >> 1 : a.T);
  const int n_pairs = (a.T + 1) >> 1, n_pp = (a.n_p + 1) >> 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(s_full + 8 * w, 1);
      mbar_init(s_empty + 8 * w, 128);
      mbar_init(p_full + 8 * w, 128);
      mbar_init(pv_done + 8 * w, 1);
    }
    for (int q = 0; q < 4; ++q) mbar_init(dec + 8 * q, 32);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 256);
    mbar_init(drain, 1);
    mbar_init(drain2, 1);
    for (int sl = 0; sl < 2; ++sl) {
      mbar_init(list_full + 8 * sl, 1);
      mbar_init(list_empty + 8 * sl, 12);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpTmaK && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kWarpMmaS) {
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
  if (threadIdx.x == 0) VSA_TR(10, 21, tmem);

  if (warp == kWarpTmaK) {
    if constexpr (C::kPair)
      producer_pair<D, NSK, true, kRef>(a, &tm_q, &tm_k, sQ, sK, k_full, k_empty, q_full, q_empty,
                                        list_full, list_empty, p_lists, p_counts, p_bm, p_cap,
                                        abort_flag, lane);
    else
      producer<R, D, NSK, true, kRef>(a, &tm_q, &tm_k, &tm_v, sQ, sK, k_full, k_empty, q_full,
                                      q_empty, s_klist, list_full, list_empty, r_items, abort_flag,
                                      lane, BH, n_v);
  } else if (warp == kWarpTmaV) {
    if constexpr (C::kPair)
      producer_pair<D, NSV, false, kRef>(a, &tm_q, &tm_v, sQ, sV, v_full, v_empty, q_full, q_empty,
                                         list_full, list_empty, p_lists, p_counts, p_bm, p_cap,
                                         abort_flag, lane);
    else
      producer<R, D, NSV, false, kRef>(a, &tm_q, &tm_v, &tm_k, sQ, sV, v_full, v_empty, q_full,
                                       q_empty, s_vlist, list_full, list_empty, r_items, abort_flag,
                                       lane, BH, n_v);
  } else if (warp == kWarpMmaS) {
    // ------------------------------------------------------------ S issuer
    // S_n = Q K_n^T into S_w (w = n & 1) as soon as K_n is in and warpgroup w
    // has read S_{n-2} out of it.  Runs ahead across items.
    if (lane == 0) {
      VSA_TL_DECL;
      uint32_t gk = 0;                   // K tiles consumed (ring position)
      uint32_t si[2] = {0, 0};           // S tiles issued per warpgroup
      uint32_t g = 0;                    // tiles of earlier items (trace only)
      int t = 0;
      bool ok = true;
      for (; ok; ++t) {
        int nk;
        if constexpr (C::kPair) {
          if (!wait_bar(list_full + 8 * (t & 1), (t >> 1) & 1, abort_flag, a.status, 24, a.wait_ns)) {
            ok = false;
            break;
          }
          if (p_counts[t & 1] < 0) break;          // no item left
          nk = (p_counts[t & 1] + 1) >> 1;
          mbar_arrive(list_empty + 8 * (t & 1));
        } else {
          if (!wait_bar(list_full + 8 * (t & 1), (t >> 1) & 1, abort_flag, a.status, 29, a.wait_ns)) {
            ok = false;
            break;
          }
          const int it = r_items[t & 1];
          if (it < 0) break;                      // no item left
          mbar_arrive(list_empty + 8 * (t & 1));
          int64_t bh;
          int i;
          decode_item(it, BH, a.n_p, n_v, bh, i);
          nk = (i < a.n_p) ? a.T : n_sink<kRef>(a) + a.k;
        }
        if (!wait_bar(q_full, t & 1, abort_flag, a.status, 5, a.wait_ns)) { ok = false; break; }
        for (int n = 0; n < nk; ++n) {
          const int w = n & 1;
          if (si[w] > 0 &&
              !wait_bar(s_empty + 8 * w, (si[w] - 1) & 1, abort_flag, a.status, 7, a.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t s = gk % NSK;
          if (!wait_bar(k_full + 8 * s, (gk / NSK) & 1, abort_flag, a.status, 6, a.wait_ns)) { ok = false; break; }
          VSA_TL(0, 'S', g + n);
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t ad = sdesc_sw128(sQ + (ks / 4) * kBM * 128 + (ks % 4) * 32, 16, 1024);
            const uint64_t bd =
                sdesc_sw128(sK + s * C::TBYTES + (ks / 4) * BN * 128 + (ks % 4) * 32, 16, 1024);
            umma_bf16(tmem + C::COL_S + w * BN, ad, bd, C::IDESC_QK, ks > 0 ? 1u : 0u);
          }
          umma_commit(s_full + 8 * w);
          umma_commit(k_empty + 8 * s);
          ++gk;
          ++si[w];
          if (n == nk - 1) umma_commit(q_empty);
        }
        g += nk;
      }
      // Drain: wait until every MMA issued above has completed.
      umma_commit(drain);
      wait_bar_drain(drain, 0);
      VSA_TR(11, 12, gk);
    }
    __syncwarp();
  } else if (warp == kWarpMmaPV) {
    // ------------------------------------------------------------ PV issuer
    // O += P_n V_n (A operand P_n from TMEM tile P_w) as soon as P_n is
    // written and V_n is in; an item's first PV also waits for the previous
    // item's epilogue to have read O.  Both warpgroups add into the one O.
    if (lane == 0) {
      VSA_TL_DECL;
      uint32_t gv = 0;                   // V tiles consumed (ring position)
      uint32_t pf[2] = {0, 0};           // p_full phases consumed per warpgroup
      uint32_t g = 0;                    // tiles of earlier items (trace only)
      int t = 0;
      bool ok = true;
      for (; ok; ++t) {
        int nk;
        if constexpr (C::kPair) {
          if (!wait_bar(list_full + 8 * (t & 1), (t >> 1) & 1, abort_flag, a.status, 25, a.wait_ns)) {
            ok = false;
            break;
          }
          if (p_counts[t & 1] < 0) break;          // no item left
          nk = (p_counts[t & 1] + 1) >> 1;
          mbar_arrive(list_empty + 8 * (t & 1));
        } else {
          if (!wait_bar(list_full + 8 * (t & 1), (t >> 1) & 1, abort_flag, a.status, 30, a.wait_ns)) {
            ok = false;
            break;
          }
          const int it = r_items[t & 1];
          if (it < 0) break;                      // no item left
          mbar_arrive(list_empty + 8 * (t & 1));
          int64_t bh;
          int i;
          decode_item(it, BH, a.n_p, n_v, bh, i);
          nk = (i < a.n_p) ? a.T : n_sink<kRef>(a) + a.k;
        }
        for (int n = 0; n < nk; ++n) {
          const int w = n & 1;
          if (n == 0 && t > 0 && !wait_bar(o_empty, (t - 1) & 1, abort_flag, a.status, 3, a.wait_ns)) {
            ok = false;
            break;
          }
          if (!wait_bar(p_full + 8 * w, pf[w] & 1, abort_flag, a.status, 4, a.wait_ns)) { ok = false; break; }
          ++pf[w];
          const uint32_t sv = gv % NSV;
          if (!wait_bar(v_full + 8 * sv, (gv / NSV) & 1, abort_flag, a.status, 12, a.wait_ns)) {
            ok = false;
            break;
          }
          VSA_TL(5, 'P', g + n);
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t bd = sdesc_sw128(sV + sv * C::TBYTES + ks * 16 * 128, BN * 128, 1024);
            umma_bf16_ts(tmem + C::COL_O, tmem + C::COL_P + w * (BN / 2) + ks * 8, bd, C::IDESC_PV,
                         (n > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(pv_done + 8 * w);
          umma_commit(v_empty + 8 * sv);
          if (n == nk - 1) umma_commit(o_full);
          ++gv;
        }
        g += nk;
      }
      umma_commit(drain2);
      wait_bar_drain(drain2, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warpgroups
    if constexpr (C::kPair) {
      // Paired 64-row tiles.  Warps 0-1 and 4-5 hold the rows of query tile
      // 2m (half 0), warps 2-3 and 6-7 those of tile 2m+1 (half 1).  A step's
      // S tile spans key tiles a = entry 2n and b = entry 2n+1 of the item's
      // list (columns [0, 64) and [64, 128)); a key tile outside this half's
      // set counts as fully masked.  The protocol is the one of the 128-row
      // kernel below (one O, a reference max shared through the mailbox,
      // lazy rescale).  Key tiles outside the set enter as -inf scores (P = 0).
      VSA_TL_DECL;
      const int wg = warp >> 2;                            // 0 or 1
      const int quad = warp & 3;
      const int half = quad >> 1;
      const int row = quad * 32 + lane;                    // = TMEM lane
      const int row_t = row - 64 * half;                   // row within the query tile
      const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
      const uint32_t col_s = C::COL_S + wg * BN;
      const uint32_t col_p = C::COL_P + wg * (BN / 2);
      const uint32_t dbar = dec + 8 * quad;
      const uint32_t s_lists =
          s_base + C::OFF_BAR + C::TAIL + 16 + 8 * ((C::bitmap_words(a.T) + 3) & ~3);
      const uint32_t s_mbox = s_base + C::OFF_X;             // reference-max mailbox [2][128]
      uint32_t G = 0;              // global index of the item's first step
      uint32_t cnt[2] = {0, 0};    // steps of each warpgroup in earlier items
      uint32_t cw = 0;             // steps processed by this warpgroup
      int t = 0;
      bool ok = true;
      for (; ok; ++t) {
        ok = __all_sync(0xFFFFFFFFu, wait_bar(list_full + 8 * (t & 1), (t >> 1) & 1, abort_flag,
                                              a.status, 26, a.wait_ns));
        if (!ok) break;
        int count, item;
        asm volatile("ld.shared.u32 %0, [%1];"
                     : "=r"(count)
                     : "r"(s_base + C::OFF_BAR + C::TAIL + 4 * (t & 1)));
        if (count < 0) break;                              // no item left
        asm volatile("ld.shared.u32 %0, [%1];"
                     : "=r"(item)
                     : "r"(s_base + C::OFF_BAR + C::TAIL + 8 + 4 * (t & 1)));
        (void)item;                                        // decoded again at the epilogue
        const int nk = (count + 1) >> 1;
        const uint32_t plist = s_lists + 4 * (t & 1) * C::list_cap(a.T);

        float m_mine = -INFINITY, l = 0.f;   // l: this warpgroup's row sum, relative to m_mine
        for (int n = wg; n < nk; n += 2, ++cw) {
          const uint32_t Gn = G + n;
          ok = __all_sync(0xFFFFFFFFu, wait_bar(s_full + 8 * wg, cw & 1, abort_flag, a.status, 8, a.wait_ns));
          if (!ok) break;
          tc_fence_after();
          // block_len of key tiles a and b for this half, 0 when outside its set
          // (an odd list ends with a zero entry)
          uint32_t ea, eb;
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(ea), "=r"(eb) : "r"(plist + 8 * n));
          const int bl2[2] = {entry_has(ea, half) ? entry_blen(ea) : 0,
                              entry_has(eb, half) ? entry_blen(eb) : 0};
          // S row into registers, then S is released at once so that S_{n+2}
          // can be issued during this step's exponentials
          // key rows past block_len of a partial key tile (rare): their score
          // columns are overwritten with -inf in TMEM, one column per store, so
          // that the row max and the exponentials below need no mask
          if (((bl2[0] | bl2[1]) & 63) != 0) mask_partial_tiles(t_lane + col_s, bl2[0], bl2[1]);
          uint32_t r[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(t_lane + col_s + 32 * c, r[c]);
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_wait_ld(r[c]);
          tc_fence_before();
          mbar_arrive(s_empty + 8 * wg);
          // a key tile outside this half's set: its scores become -inf in
          // registers, so that the row max, the exponentials (exp2(-inf) = 0)
          // and the row sums below run one branch-free code path for both
          // query tiles of the pair
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            if (bl2[c2] == 0) {                              // warp-uniform
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 32; ++e) r[2 * c2 + h][e] = __float_as_uint(-INFINITY);
            }
          }
          // row max over raw scores (scale > 0 commutes with max), four chains
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int e = 0; e < 32; e += 2)
                mx4[(e >> 1) & 3] = fmax3(mx4[(e >> 1) & 3], __uint_as_float(r[2 * c2 + h][e]),
                                          __uint_as_float(r[2 * c2 + h][e + 1]));
          }
          const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]);
          // m_ref after step n-1 (the previous global step's decision; an
          // item's first step starts from -inf), then this step's decision
          float m_prev = -INFINITY;
          if (Gn > 0) {
            ok = __all_sync(0xFFFFFFFFu, wait_bar(dbar, (Gn - 1) & 1, abort_flag, a.status, 14, a.wait_ns));
            if (!ok) break;
            if (n > 0) asm volatile("ld.shared.f32 %0, [%1];" : "=f"(m_prev) : "r"(s_mbox + 4 * (((Gn - 1) & 1) * 128 + row)));
          }
          const float m_cand = fmaxf(m_prev, mx * a.scale_log2);
          const bool rescale = __any_sync(0xFFFFFFFFu, m_cand > m_prev + 8.0f);
          const float m_new = rescale ? m_cand : m_prev;
          if (m_new != -INFINITY) {
            // this warpgroup's row sum follows the reference max (-inf only
            // while no key of the item has reached these rows)
            l *= ex2(m_mine - m_new);
            m_mine = m_new;
          }
          // P_w is free once this warpgroup's previous PV is complete
          if (cw > 0) {
            ok = __all_sync(0xFFFFFFFFu,
                            wait_bar(pv_done + 8 * wg, (cw - 1) & 1, abort_flag, a.status, 9, a.wait_ns));
            if (!ok) break;
          }
          tc_fence_after();
          bool published = false;            // warp-uniform
          {
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const uint64_t sc2 = f2pack(a.scale_log2, a.scale_log2), nm2 = f2pack(-m_use, -m_use);
            uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              if (c2 == 1 && kPubChunk > 0 && kPubChunk < 4) {
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(s_mbox + 4 * ((Gn & 1) * 128 + row)), "f"(m_new) : "memory");
                mbar_arrive(dbar);
                published = true;
              }
              // P in 16-column stores, so that only 16 packed words are live
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t pw[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                  float x0, x1;
                  f2unpack(ffma2(f2pack(__uint_as_float(r[2 * c2 + h][e]),
                                        __uint_as_float(r[2 * c2 + h][e + 1])),
                                 sc2, nm2),
                           x0, x1);
                  const float p0 = ex2(x0), p1 = ex2(x1);
                  acc2[(e >> 1) & 1] = fadd2(acc2[(e >> 1) & 1], f2pack(p0, p1));
                  pw[e >> 1] = pack_bf16(p0, p1);
                }
                tmem_st16(t_lane + col_p + 32 * c2 + 16 * h, pw);
              }
            }
            float s0, s1;
            f2unpack(fadd2(acc2[0], acc2[1]), s0, s1);
            l += s0 + s1;
          }
          if (!published) {
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(s_mbox + 4 * ((Gn & 1) * 128 + row)), "f"(m_new) : "memory");
            mbar_arrive(dbar);
          }
          // O rescale when the reference max moved: O holds PV_0..PV_{n-1}
          // relative to m_prev; PV_{n-1} (the partner's step) must be complete,
          // and PV_n is not issued before the p_full arrival below.
          if (rescale && n > 0) {
            const uint32_t idx = cnt[1 - wg] + uint32_t((n - 1) >> 1);
            ok = __all_sync(0xFFFFFFFFu,
                            wait_bar(pv_done + 8 * (1 - wg), idx & 1, abort_flag, a.status, 15, a.wait_ns));
            if (!ok) break;
            tc_fence_after();
            const float alpha = ex2(m_prev - m_new);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(t_lane + C::COL_O + 32 * c, o);
              tmem_wait_ld(o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(t_lane + C::COL_O + 32 * c, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_full + 8 * wg);
        }
        if (!ok) break;
        // ---- epilogue (as in the 128-row kernel), per query tile of the pair
        ok = __all_sync(0xFFFFFFFFu, wait_bar(o_full, t & 1, abort_flag, a.status, 10, a.wait_ns));
        if (!ok) break;
        cnt[0] += uint32_t((nk + 1) / 2);
        cnt[1] += uint32_t(nk / 2);
        tc_fence_after();
        x_m[wg * 128 + row] = m_mine;
        x_l[wg * 128 + row] = l;
        if (*abort_flag) { ok = false; break; }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        // the item (re-read from its slot: not kept in registers through the steps)
        asm volatile("ld.shared.u32 %0, [%1];"
                     : "=r"(item)
                     : "r"(s_base + C::OFF_BAR + C::TAIL + 8 + 4 * (t & 1)));
        int64_t bh;
        int m;
        decode_pair(item, BH, n_pp, n_pairs, bh, m);
        const int i = 2 * m + half;                         // this warp's query tile
        const bool rows_active = i < a.T;                   // warp-uniform
        const int q_live = rows_active ? __ldg(a.block_len + i) : 0;
        if (rows_active) {
          const float m0 = x_m[row], m1 = x_m[128 + row];
          const float l0 = x_l[row], l1 = x_l[128 + row];
          const float mm = fmaxf(m0, m1);
          const float lt = (l0 > 0.f ? l0 * ex2(m0 - mm) : 0.f) + (l1 > 0.f ? l1 * ex2(m1 - mm) : 0.f);
          const bool live = row_t < q_live;
          const float inv = live ? 1.0f / lt : 0.f;
          const bool fused = a.gate != nullptr;
          const int64_t tok =
              (fused && live) ? int64_t(__ldg(a.row_src + int64_t(i) * R + row_t)) : 0;
          uint16_t* orow = fused ? a.out + (bh * a.n_tok + tok) * D + wg * (D / 2)
                                 : a.out + (bh * a.n_pad + int64_t(i) * R + row_t) * D + wg * (D / 2);
          const uint16_t* grow = fused ? a.gate + (bh * a.n_tok + tok) * D + wg * (D / 2) : nullptr;
          const float* ocrow = fused ? a.o_coarse + (bh * a.T + i) * D + wg * (D / 2) : nullptr;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            tmem_ld32(t_lane + C::COL_O + wg * (D / 2) + 32 * c, o);
            tmem_wait_ld(o);
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(o[8 * q + e]) * inv;
              if (fused) {
                if (!live) continue;                  // pad rows have no natural token
                const uint4 gv = __ldg(reinterpret_cast<const uint4*>(grow + 32 * c + 8 * q));
                const float4 c0v = __ldg(reinterpret_cast<const float4*>(ocrow + 32 * c + 8 * q));
                const float4 c1v = __ldg(reinterpret_cast<const float4*>(ocrow + 32 * c + 8 * q + 4));
                const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                const float cv[8] = {c0v.x, c0v.y, c0v.z, c0v.w, c1v.x, c1v.y, c1v.z, c1v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  v[2 * e] = fmaf(sigmoid_fast(__uint_as_float(gw[e] << 16)), cv[2 * e], v[2 * e]);
                  v[2 * e + 1] = fmaf(sigmoid_fast(__uint_as_float(gw[e] & 0xFFFF0000u)),
                                      cv[2 * e + 1], v[2 * e + 1]);
                }
              }
              uint4 u;
              u.x = pack_bf16(v[0], v[1]);
              u.y = pack_bf16(v[2], v[3]);
              u.z = pack_bf16(v[4], v[5]);
              u.w = pack_bf16(v[6], v[7]);
              dst[q] = u;
            }
          }
          if (a.lse != nullptr && wg == 0)
            a.lse[bh * a.n_pad + int64_t(i) * R + row_t] =
                live ? (mm + __log2f(lt)) * 0.69314718055994531f : 0.f;
        }
        tc_fence_before();
        mbar_arrive(o_empty);
        __syncwarp();
        if (lane == 0) mbar_arrive(list_empty + 8 * (t & 1));   // this warp is done with the list
        G += nk;
      }
    } else {
      // Warpgroup wg takes the tiles n = wg (mod 2) of an item; both add into
      // one O, scaled by one reference max m_ref per row.  m_ref after tile n is
      // decided by the warp that runs tile n from m_ref after tile n-1 (read
      // from the mailbox its partner warp on the same TMEM lanes wrote) and its
      // own row max, and published in turn; it moves only when a row grew by
      // more than 2^8 (exact: p <= 256), and then that warp rescales its O rows
      // once PV_{n-1} is complete.
      VSA_TL_DECL;
      const int wg = warp >> 2;                            // 0 or 1
      const int quad = warp & 3;
      const bool rows_active = (R == 128) || (quad < 2);
      const int row = quad * 32 + lane;                    // = TMEM lane
      const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
      const uint32_t col_s = C::COL_S + wg * BN;
      const uint32_t col_p = C::COL_P + wg * (BN / 2);
      const uint32_t dbar = dec + 8 * quad;
      uint32_t G = 0;              // global index of the item's first tile
      uint32_t cnt[2] = {0, 0};    // tiles of each warpgroup in earlier items
      uint32_t cw = 0;             // tiles processed by this warpgroup
      int t = 0;
      bool ok = true;
      for (; ok; ++t) {
        ok = __all_sync(0xFFFFFFFFu, wait_bar(list_full + 8 * (t & 1), (t >> 1) & 1, abort_flag,
                                              a.status, 31, a.wait_ns));
        if (!ok) break;
        const int item = r_items[t & 1];
        if (item < 0) break;                               // no item left
        int64_t bh;
        int i;
        decode_item(item, BH, a.n_p, n_v, bh, i);
        const bool dense = i < a.n_p;
        const int nk = dense ? a.T : n_sink<kRef>(a) + a.k;
        // Group barrier of the 256 softmax threads around the per-item list.  A
        // warp that sees the abort flag leaves instead: the others then also see
        // it before they could block here (they wait on the same mbarrier phases
        // first).
        if (*abort_flag) { ok = false; break; }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        for (int x = threadIdx.x; x < nk; x += 256) {
          const int j = step_tile_global<kRef>(a, bh, i, dense, x);
          s_blen[x] = uint8_t(__ldg(a.block_len + j) - 1);
        }
        if (*abort_flag) { ok = false; break; }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const int q_live = __ldg(a.block_len + i);

        float m_mine = -INFINITY, l = 0.f;   // l: this warpgroup's row sum, relative to m_mine
        for (int n = wg; n < nk; n += 2, ++cw) {
          const uint32_t Gn = G + n;
          if (lane == 0) VSA_TR(quad + 4 * wg, 13, Gn);
          if (threadIdx.x % 128 == 0) VSA_TL(1 + wg, 'a', Gn);
          ok = __all_sync(0xFFFFFFFFu, wait_bar(s_full + 8 * wg, cw & 1, abort_flag, a.status, 8, a.wait_ns));
          if (!ok) break;
          if (threadIdx.x % 128 == 0) VSA_TL(1 + wg, 's', Gn);
          tc_fence_after();
          // key rows past block_len (a partial key tile, rare): -inf in TMEM
          if (rows_active && int(s_blen[n]) + 1 < BN) mask_tile_tail(t_lane + col_s, int(s_blen[n]) + 1);
          uint32_t r[BN / 32][32];
          if (rows_active) {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_lane + col_s + 32 * c, r[c]);
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_wait_ld(r[c]);
          }
          tc_fence_before();
          mbar_arrive(s_empty + 8 * wg);
          if (threadIdx.x % 128 == 0) VSA_TL(1 + wg, 'l', Gn);
          // row max over raw scores (scale > 0 commutes with max), four chains
          float mx = -INFINITY;
          if (rows_active) {
            float mx4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) mx4[q] = -INFINITY;
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
#pragma unroll
              for (int e = 0; e < 32; e += 2)
                mx4[(e >> 1) & 3] = fmax3(mx4[(e >> 1) & 3], __uint_as_float(r[c][e]),
                                          __uint_as_float(r[c][e + 1]));
            mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]);
          }
          // m_ref after tile n-1 (the previous global tile's decision; an item's
          // first tile starts from -inf), then this tile's decision
          float m_prev = -INFINITY;
          if (Gn > 0) {
            ok = __all_sync(0xFFFFFFFFu, wait_bar(dbar, (Gn - 1) & 1, abort_flag, a.status, 14, a.wait_ns));
            if (!ok) break;
            if (n > 0) m_prev = mbox[((Gn - 1) & 1) * 128 + row];
          }
          const float m_cand = fmaxf(m_prev, mx * a.scale_log2);
          // warp-uniform (the O rescale below uses warp-collective TMEM access)
          const bool rescale = __any_sync(0xFFFFFFFFu, m_cand > m_prev + 8.0f);
          const float m_new = rescale ? m_cand : m_prev;
          bool published = false;            // warp-uniform
          if (threadIdx.x % 128 == 0) VSA_TL(1 + wg, 'm', Gn);
          if (rows_active) {
            // this warpgroup's row sum follows the reference max
            l *= ex2(m_mine - m_new);
            m_mine = m_new;
          }
          // P_w is free once this warpgroup's previous PV is complete
          if (cw > 0) {
            ok = __all_sync(0xFFFFFFFFu,
                            wait_bar(pv_done + 8 * wg, (cw - 1) & 1, abort_flag, a.status, 9, a.wait_ns));
            if (!ok) break;
          }
          tc_fence_after();
          if (rows_active) {
            // exponentials on pairs: packed scale-and-subtract, two exp2, packed
            // row sums, P packed to bf16 and stored to P_w every 64 scores.  One
            // exponential in kExp2FmaShare runs on the FMA pipe.
            const uint64_t sc2 = f2pack(a.scale_log2, a.scale_log2), nm2 = f2pack(-m_new, -m_new);
            uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c2 = 0; c2 < BN / 64; ++c2) {
              uint32_t pw[32];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c = 2 * c2 + h;
                if (kPubChunk > 0 && kPubChunk < BN / 32 && c == kPubChunk) {
                  mbox[(Gn & 1) * 128 + row] = m_new;
                  mbar_arrive(dbar);
                  published = true;
                }
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                  float x0, x1;
                  f2unpack(ffma2(f2pack(__uint_as_float(r[c][e]), __uint_as_float(r[c][e + 1])), sc2,
                                 nm2),
                           x0, x1);
                  const bool fma0 = kExp2FmaShare > 0 && e % kExp2FmaShare == kExp2FmaShare - 1;
                  const bool fma1 = kExp2FmaShare > 0 && (e + 1) % kExp2FmaShare == kExp2FmaShare - 1;
                  const float p0 = fma0 ? exp2_fma(x0) : ex2(x0);
                  const float p1 = fma1 ? exp2_fma(x1) : ex2(x1);
                  acc2[(e >> 1) & 3] = fadd2(acc2[(e >> 1) & 3], f2pack(p0, p1));
                  pw[16 * h + (e >> 1)] = pack_bf16(p0, p1);
                }
              }
              tmem_st32(t_lane + col_p + 32 * c2, pw);
            }
            float s0, s1, s2, s3;
            f2unpack(fadd2(acc2[0], acc2[1]), s0, s1);
            f2unpack(fadd2(acc2[2], acc2[3]), s2, s3);
            l += (s0 + s1) + (s2 + s3);
          }
          // Publish the decision only now: the partner warp, which shares this
          // warp's SM sub-partition and its MUFU unit, cannot start its own
          // exponentials before ours are done, so the two warps take turns on
          // the MUFU and each does its loads, max and stores during the
          // other's exponentials.
          if (!published) {
            mbox[(Gn & 1) * 128 + row] = m_new;
            mbar_arrive(dbar);
          }
          if (threadIdx.x % 128 == 0) VSA_TL(1 + wg, 'w', Gn);
          // O rescale when the reference max moved: O holds PV_0..PV_{n-1}
          // relative to m_prev; PV_{n-1} (the partner's tile) must be complete,
          // and PV_n is not issued before the p_full arrival below.
          if (rescale && n > 0) {
            const uint32_t idx = cnt[1 - wg] + uint32_t((n - 1) >> 1);
            ok = __all_sync(0xFFFFFFFFu,
                            wait_bar(pv_done + 8 * (1 - wg), idx & 1, abort_flag, a.status, 15, a.wait_ns));
            if (!ok) break;
            tc_fence_after();
            if (rows_active) {
              const float alpha = ex2(m_prev - m_new);
#pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(t_lane + C::COL_O + 32 * c, o);
                tmem_wait_ld(o);
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st32(t_lane + C::COL_O + 32 * c, o);
              }
            }
          }
          if (rows_active) tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_full + 8 * wg);
          if (lane == 0) VSA_TR(quad + 4 * wg, 16, Gn);
          if (threadIdx.x % 128 == 0) VSA_TL(1 + wg, 'W', Gn);
        }
        if (!ok) break;
        // ---- epilogue: once every PV of the item is complete (o_full), add the
        // two row sums (each relative to its warpgroup's last reference max; O
        // is relative to the larger) and store O / l (warpgroup wg: columns
        // [wg*D/2, (wg+1)*D/2)), fused with the gated combine when a gate is given.
        const uint32_t g_last = G + nk - 1;
        (void)g_last;
        if (lane == 0) VSA_TR(quad + 4 * wg, 17, g_last);
        ok = __all_sync(0xFFFFFFFFu, wait_bar(o_full, t & 1, abort_flag, a.status, 10, a.wait_ns));
        if (!ok) break;
        cnt[0] += uint32_t((nk + 1) / 2);
        cnt[1] += uint32_t(nk / 2);
        tc_fence_after();
        x_m[wg * 128 + row] = m_mine;
        x_l[wg * 128 + row] = l;
        if (*abort_flag) { ok = false; break; }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (rows_active) {
          const float m0 = x_m[row], m1 = x_m[128 + row];
          const float l0 = x_l[row], l1 = x_l[128 + row];
          const float mm = fmaxf(m0, m1);
          const float lt = (l0 > 0.f ? l0 * ex2(m0 - mm) : 0.f) + (l1 > 0.f ? l1 * ex2(m1 - mm) : 0.f);
          const bool live = row < q_live;
          const float inv = live ? 1.0f / lt : 0.f;
          const bool fused = a.gate != nullptr;
          const int64_t tok = (fused && live) ? int64_t(__ldg(a.row_src + int64_t(i) * R + row)) : 0;
          uint16_t* orow = fused ? a.out + (bh * a.n_tok + tok) * D + wg * (D / 2)
                                 : a.out + (bh * a.n_pad + int64_t(i) * R + row) * D + wg * (D / 2);
          const uint16_t* grow = fused ? a.gate + (bh * a.n_tok + tok) * D + wg * (D / 2) : nullptr;
          const float* ocrow = fused ? a.o_coarse + (bh * a.T + i) * D + wg * (D / 2) : nullptr;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            tmem_ld32(t_lane + C::COL_O + wg * (D / 2) + 32 * c, o);
            tmem_wait_ld(o);
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(o[8 * q + e]) * inv;
              if (fused) {
                if (!live) continue;                  // pad rows have no natural token
                const uint4 gv =
                    VSA_STREAM_IO ? __ldcs(reinterpret_cast<const uint4*>(grow + 32 * c + 8 * q))
                                  : __ldg(reinterpret_cast<const uint4*>(grow + 32 * c + 8 * q));
                const float4 c0v = __ldg(reinterpret_cast<const float4*>(ocrow + 32 * c + 8 * q));
                const float4 c1v = __ldg(reinterpret_cast<const float4*>(ocrow + 32 * c + 8 * q + 4));
                const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                const float cv[8] = {c0v.x, c0v.y, c0v.z, c0v.w, c1v.x, c1v.y, c1v.z, c1v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  v[2 * e] = fmaf(sigmoid_fast(__uint_as_float(gw[e] << 16)), cv[2 * e], v[2 * e]);
                  v[2 * e + 1] =
                      fmaf(sigmoid_fast(__uint_as_float(gw[e] & 0xFFFF0000u)), cv[2 * e + 1], v[2 * e + 1]);
                }
              }
              uint4 u;
              u.x = pack_bf16(v[0], v[1]);
              u.y = pack_bf16(v[2], v[3]);
              u.z = pack_bf16(v[4], v[5]);
              u.w = pack_bf16(v[6], v[7]);
              if (VSA_STREAM_IO)
                __stcs(dst + q, u);
              else
                dst[q] = u;
            }
          }
          if (a.lse != nullptr && wg == 0)
            a.lse[bh * a.n_pad + int64_t(i) * R + row] =
                live ? (mm + __log2f(lt)) * 0.69314718055994531f : 0.f;
        }
        tc_fence_before();
        mbar_arrive(o_empty);
        __syncwarp();
        if (lane == 0) mbar_arrive(list_empty + 8 * (t & 1));   // this warp is done with the item
        if (lane == 0) VSA_TR(quad + 4 * wg, 18, g_last);
        G += nk;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  if (lane == 0) VSA_TR(warp, 19, 0);
  tc_fence_before();
  __syncthreads();
  // the last CTA to finish resets the work counter for the next launch (no
  // CTA takes an item once it has counted itself done)
  if (threadIdx.x == 0 && atomicAdd(a.work + 1, 1u) == gridDim.x - 1) {
    atomicExch(a.work, 0u);
    atomicExch(a.work + 1, 0u);
  }
  if (warp == kWarpMmaS) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
    if (lane == 0) VSA_TR(12, 20, 0);
  }
}

// ---------------------------------------------------------------- host side

// Dynamic shared memory of one CTA (+1 KB so the kernel can align its base to
// 1024 bytes), at least 120 KB so that two CTAs never share an SM (each holds
// its TMEM columns for its whole lifetime).
constexpr size_t kMaxSmem = 227 * 1024;
template <int R, int D>
size_t attn_smem_bytes(int T, int k) {
  const size_t need = Cfg<R, D>::bytes(T, k) + 1024;
  return need < size_t(120 * 1024) ? size_t(120 * 1024) : need;
}

template <int R, int D>
vsa_status launch_rd(const vsa_plan_s* p, const void* q_t, const void* k_t, const void* v_t,
                     const int32_t* topk_idx, int64_t bh, int k, float scale, void* out,
                     float* lse_t, const void* gate, const float* o_coarse, const int32_t* topk_ref,
                     int k_ref, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes<R, D>(p->n_tiles, k);
  if (smem > kMaxSmem)
    return fail(VSA_ERR_UNSUPPORTED, "too many tiles for the sparse attention kernel's lists");
  const int64_t rows = bh * p->n_padded;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q_t, rows, D, kBM) || !make_map(&mk, k_t, rows, D, R) ||
      !make_map(&mv, v_t, rows, D, R))
    return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  const bool thin = k_ref >= 0;
  auto kernel = thin ? sparse_attn_kernel<R, D, true> : sparse_attn_kernel<R, D, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, cudaGetErrorString(e));
  AttnArgs a;
  a.topk = topk_idx;
  a.block_len = p->d_block_len;
  a.out = static_cast<uint16_t*>(out);
  a.gate = static_cast<const uint16_t*>(gate);
  a.o_coarse = o_coarse;
  a.row_src = p->d_row_src;
  a.n_tok = p->n_tokens;
  a.lse = lse_t;
  a.status = p->d_status;
  a.wait_ns = wait_limit_ns();
  a.work = p->d_status + 4;
  a.T = p->n_tiles;
  a.n_p = p->n_prefix_tiles;
  a.k = k;
  // k_ref < 0: every reference tile is a sink; else the k_ref listed ones
  a.topk_ref = thin ? topk_ref : nullptr;
  a.k_ref = thin ? k_ref : 0;
  a.n_sink = thin ? k_ref : p->n_prefix_tiles;
  a.n_pad = p->n_padded;
  a.scale_log2 = scale * 1.4426950408889634f;
  // 64-row tiles: one item per pair of consecutive query tiles
  const int64_t items = bh * (Cfg<R, D>::kPair ? (p->n_tiles + 1) / 2 : p->n_tiles);
  if (items >= (int64_t(1) << 31)) return fail(VSA_ERR_UNSUPPORTED, "too many work items");
  a.n_items = int(items);
  a.BH = int(bh);
  const int grid = int(std::min<int64_t>(items, p->num_sms > 0 ? p->num_sms : 148));
  kernel<<<grid, kThreadsAttn, smem, stream>>>(mq, mk, mv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, std::string("sparse_attn launch: ") + cudaGetErrorString(e));
  return VSA_OK;
}

}  // namespace

vsa_status launch_sparse_attn(const vsa_plan_s* p, const void* q_t, const void* k_t,
                              const void* v_t, const int32_t* topk_idx, int64_t bh, int D, int k,
                              float scale, void* out, float* lse_t, const void* gate,
                              const float* o_coarse, const int32_t* topk_ref, int k_ref,
                              cudaStream_t stream) {
  if (p->n_padded * bh >= (int64_t(1) << 31))
    return fail(VSA_ERR_UNSUPPORTED, "B*H*N_pad rows exceed the 32-bit TMA coordinate range");
  if (p->R == 128) {
    if (D == 128)
      return launch_rd<128, 128>(p, q_t, k_t, v_t, topk_idx, bh, k, scale, out, lse_t, gate,
                                 o_coarse, topk_ref, k_ref, stream);
    return launch_rd<128, 64>(p, q_t, k_t, v_t, topk_idx, bh, k, scale, out, lse_t, gate, o_coarse,
                              topk_ref, k_ref, stream);
  }
  if (D == 128)
    return launch_rd<64, 128>(p, q_t, k_t, v_t, topk_idx, bh, k, scale, out, lse_t, gate, o_coarse,
                              topk_ref, k_ref, stream);
  return launch_rd<64, 64>(p, q_t, k_t, v_t, topk_idx, bh, k, scale, out, lse_t, gate, o_coarse,
                           topk_ref, k_ref, stream);
}

}  // namespace vsa
