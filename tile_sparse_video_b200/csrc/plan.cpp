// Host planner: token -> padded-row permutation and the tile table.
//
// Source: "ComfyUI-Ref2VA-VSA proves a sparse attention gate can be
// transplanted ..." (SnackOnAI), "The Code, Annotated", snippet one: every
// prefix segment is cut into R-row tiles, its last tile may be short, and each
// segment starts a fresh tile, so no tile mixes modalities; the video follows,
// flattened t-major then h then w, cut into cubes visited t0, h0, w0.  Cubes at
// the far edge of a grid whose extent is not a multiple of the cube extent are
// clipped (this reproduces the page's "It In Action" count of 660 video tiles
// and 43,904 rows for a 37 x 24 x 42 grid).  Inside a cube tokens are laid out
// in lexicographic (t, h, w) order at the head of the tile; pad rows follow.
//
// The planner writes each token's row directly from its coordinates (one pass
// per cube, contiguous runs along w) and then verifies the result the way the
// page's guard rails do: injective, every token placed once, each tile holding
// a single segment.
#include <algorithm>
#include <cstring>

#include "vsa_internal.h"

namespace vsa {

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

vsa_status build_plan(const vsa_geometry& g, vsa_plan_s* p) {
  const int64_t tt = g.tile_t, th = g.tile_h, tw = g.tile_w;
  const int64_t Tg = g.grid_t, Hg = g.grid_h, Wg = g.grid_w;
  if (tt <= 0 || th <= 0 || tw <= 0)
    return fail(VSA_ERR_INVALID_ARG, "tile extents must be positive");
  if (Tg < 0 || Hg < 0 || Wg < 0)
    return fail(VSA_ERR_PLAN, "video grid extents must be >= 0");
  if (g.n_prefix_segments < 0 || (g.n_prefix_segments > 0 && g.prefix_lens == nullptr))
    return fail(VSA_ERR_INVALID_ARG, "prefix_lens is NULL");
  const int64_t R = tt * th * tw;
  if (R != 64 && R != 128)
    return fail(VSA_ERR_UNSUPPORTED, "tile rows R = tile_t*tile_h*tile_w must be 64 or 128");

  int64_t P = 0, n_p = 0;
  for (int s = 0; s < g.n_prefix_segments; ++s) {
    if (g.prefix_lens[s] < 0) return fail(VSA_ERR_PLAN, "negative prefix segment length");
    P += g.prefix_lens[s];
    n_p += ceil_div(g.prefix_lens[s], R);
  }
  const int64_t cT = ceil_div(Tg, tt), cH = ceil_div(Hg, th), cW = ceil_div(Wg, tw);
  const int64_t n_v = cT * cH * cW;
  const int64_t N = P + Tg * Hg * Wg;
  const int64_t T = n_p + n_v;
  if (T * R >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return fail(VSA_ERR_UNSUPPORTED, "sequence too long for 32-bit row indices");

  p->R = int(R);
  p->n_tokens = N;
  p->n_tiles = int(T);
  p->n_prefix_tiles = int(n_p);
  p->n_padded = T * R;
  p->untile.assign(size_t(N), -1);
  p->row_src.assign(size_t(T * R), -1);
  p->block_len.assign(size_t(T), 0);
  p->tile_seg.assign(size_t(T), -1);

  // Prefix: segment s fills ceil(L/R) tiles of its own.
  int64_t tok = 0, tile = 0;
  for (int s = 0; s < g.n_prefix_segments; ++s) {
    for (int64_t j = 0; j < g.prefix_lens[s]; ++j) {
      const int64_t t = tile + j / R;
      p->untile[size_t(tok + j)] = int32_t(t * R + j % R);
    }
    const int64_t ntile = ceil_div(g.prefix_lens[s], R);
    for (int64_t c = 0; c < ntile; ++c) {
      p->block_len[size_t(tile + c)] = int32_t(std::min(R, g.prefix_lens[s] - c * R));
      p->tile_seg[size_t(tile + c)] = s;
    }
    tok += g.prefix_lens[s];
    tile += ntile;
  }

  // Video cubes, in cube order t0, h0, w0.
  for (int64_t ct = 0; ct < cT; ++ct)
    for (int64_t ch = 0; ch < cH; ++ch)
      for (int64_t cw = 0; cw < cW; ++cw) {
        const int64_t t0 = ct * tt, h0 = ch * th, w0 = cw * tw;
        const int64_t bt = std::min(tt, Tg - t0), bh = std::min(th, Hg - h0),
                      bw = std::min(tw, Wg - w0);
        const int64_t cube = n_p + (ct * cH + ch) * cW + cw;
        int64_t slot = 0;
        for (int64_t a = 0; a < bt; ++a)
          for (int64_t b = 0; b < bh; ++b) {
            const int64_t base = P + ((t0 + a) * Hg + (h0 + b)) * Wg + w0;
            for (int64_t c = 0; c < bw; ++c, ++slot)
              p->untile[size_t(base + c)] = int32_t(cube * R + slot);
          }
        p->block_len[size_t(cube)] = int32_t(bt * bh * bw);
      }

  // Guard rails: injective, every token placed once, one segment per tile.
  for (int64_t n = 0; n < N; ++n) {
    const int32_t r = p->untile[size_t(n)];
    if (r < 0 || r >= T * R) return fail(VSA_ERR_PLAN, "token left unplaced");
    if (p->row_src[size_t(r)] != -1) return fail(VSA_ERR_PLAN, "untile map is not injective");
    p->row_src[size_t(r)] = int32_t(n);
  }
  std::vector<int32_t> seg_of_token(size_t(N), -1);
  {
    int64_t o = 0;
    for (int s = 0; s < g.n_prefix_segments; ++s)
      for (int64_t j = 0; j < g.prefix_lens[s]; ++j) seg_of_token[size_t(o++)] = s;
  }
  for (int64_t t = 0; t < T; ++t) {
    const int32_t bl = p->block_len[size_t(t)];
    if (bl < 1 || bl > R) return fail(VSA_ERR_PLAN, "empty or overfull tile");
    for (int64_t r = 0; r < R; ++r) {
      const int32_t src = p->row_src[size_t(t * R + r)];
      if ((src >= 0) != (r < bl)) return fail(VSA_ERR_PLAN, "live rows are not at the tile head");
      if (src >= 0 && seg_of_token[size_t(src)] != p->tile_seg[size_t(t)])
        return fail(VSA_ERR_PLAN, "tile mixes segments");
    }
  }
  return VSA_OK;
}

}  // namespace vsa
