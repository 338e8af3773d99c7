// Token blocks of the latent video grid (T, Hg, Wg), tokens in raster order
// n = (t * Hg + y) * Wg + x.
//
// A block is either a run of `block` consecutive tokens (tw == 0; the last run
// may be short), or a 3-D tile of tt x th x tw tokens (tiles cover the grid
// exactly; tile (it, iy, ix) is block (it * nty + iy) * ntx + ix, and inside a
// tile the tokens are taken in raster order of (dt, dy, dx)).  Tiles are one of
// the selection's open choices: Sol-Attn decides per query which parts of the
// attention matter (ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan
// afspelen", section "Waar de snelheidswinst vandaan komt") without saying
// what a part is.
#pragma once

namespace sol {

struct BlockMap {
  int block;          // tokens per block (tt * th * tw when tiled)
  int tt, th, tw;     // tile extents; tw == 0: runs of consecutive tokens
  int gh, gw;         // grid rows and columns
  int nty, ntx;       // tiles per frame column and row (tiled only)
};

__host__ __device__ __forceinline__ BlockMap raster_blocks(int block, int gh, int gw) {
  return BlockMap{block, 0, 0, 0, gh, gw, 0, 0};
}

__host__ __device__ __forceinline__ BlockMap tiled_blocks(int tt, int th, int tw, int gh, int gw) {
  return BlockMap{tt * th * tw, tt, th, tw, gh, gw, gh / th, gw / tw};
}

// Grid coordinates of the first token of tiled block `blk`.
__host__ __device__ __forceinline__ void tile_origin(const BlockMap& m, int blk, int& t0, int& y0, int& x0) {
  x0 = (blk % m.ntx) * m.tw;
  y0 = ((blk / m.ntx) % m.nty) * m.th;
  t0 = (blk / (m.ntx * m.nty)) * m.tt;
}

// Token index of the l-th token of block `blk` (l < block, and for runs l < the run's length).
__host__ __device__ __forceinline__ int block_token(const BlockMap& m, int blk, int l) {
  if (m.tw == 0) return blk * m.block + l;
  int t0, y0, x0;
  tile_origin(m, blk, t0, y0, x0);
  const int dx = l % m.tw, dy = (l / m.tw) % m.th, dt = l / (m.tw * m.th);
  return ((t0 + dt) * m.gh + y0 + dy) * m.gw + x0 + dx;
}

// Block holding token n.
__host__ __device__ __forceinline__ int token_block(const BlockMap& m, int n) {
  if (m.tw == 0) return n / m.block;
  const int hw = m.gh * m.gw;
  const int t = n / hw, y = (n / m.gw) % m.gh, x = n % m.gw;
  return ((t / m.tt) * m.nty + y / m.th) * m.ntx + x / m.tw;
}

// Position of token n inside its block.
__host__ __device__ __forceinline__ int token_slot(const BlockMap& m, int n) {
  if (m.tw == 0) return n % m.block;
  const int hw = m.gh * m.gw;
  const int t = n / hw, y = (n / m.gw) % m.gh, x = n % m.gw;
  return ((t % m.tt) * m.th + y % m.th) * m.tw + x % m.tw;
}

}  // namespace sol
