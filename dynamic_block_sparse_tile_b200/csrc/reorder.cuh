// Token reorder between raster order and 3-D tile order ("Fractal Flattening"
// on the NABLA page, section "Méthodologie : NABLA").  Pure permutation of
// 16-byte chunks; HBM-bound.  One thread moves one 16-byte chunk of a token
// row per iteration; consecutive threads cover consecutive chunks of the same
// tiled row, so both the gather side (runs of tx raster tokens) and the
// scatter side are coalesced.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace dbst {

struct TileGeo {
  int N;              // tokens per (b, h)
  int X, Y;           // token grid (X fastest)
  int tt, ty, tx;     // tile shape
  int nX, nY;         // tiles per row / column
};

__device__ __forceinline__ int tiled_to_raster(int r, const TileGeo& g) {
  const int tile = r >> 6, off = r & 63;
  const int Tx = tile % g.nX;
  const int tq = tile / g.nX;
  const int Ty = tq % g.nY;
  const int Tt = tq / g.nY;
  const int dx = off % g.tx;
  const int oq = off / g.tx;
  const int dy = oq % g.ty;
  const int dt = oq / g.ty;
  return ((Tt * g.tt + dt) * g.Y + (Ty * g.ty + dy)) * g.X + (Tx * g.tx + dx);
}

constexpr int kPermuteUnroll = 4;   // 16-byte chunks in flight per thread

// to_tiled = 1: dst[tiled r] = src[raster n(r)];  0: dst[raster n(r)] = src[tiled r].
// grid.y = (b, h) pair; each CTA moves 256 * kPermuteUnroll consecutive chunks of that head,
// thread t handling chunks t, t + 256, ... so every load is issued before the first store.
template <int CPR_LOG2>
__global__ void __launch_bounds__(256) tile_permute_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           TileGeo g, int to_tiled) {
  constexpr int CPR = 1 << CPR_LOG2;   // 16-byte chunks per token row
  const long long head = static_cast<long long>(blockIdx.y) * g.N;
  const int total = g.N << CPR_LOG2;   // chunks in this head
  const int c0 = blockIdx.x * (256 * kPermuteUnroll) + threadIdx.x;
  uint4 v[kPermuteUnroll];
  long long dsto[kPermuteUnroll];
#pragma unroll
  for (int e = 0; e < kPermuteUnroll; ++e) {
    const int c = c0 + 256 * e;
    dsto[e] = -1;
    if (c < total) {
      const int r = c >> CPR_LOG2, ch = c & (CPR - 1);
      const int n = tiled_to_raster(r, g);
      const long long tiled_off = ((head + r) << CPR_LOG2) + ch;
      const long long raster_off = ((head + n) << CPR_LOG2) + ch;
      v[e] = ld_stream(src + (to_tiled ? raster_off : tiled_off));
      dsto[e] = to_tiled ? tiled_off : raster_off;
    }
  }
#pragma unroll
  for (int e = 0; e < kPermuteUnroll; ++e)
    if (dsto[e] >= 0) dst[dsto[e]] = v[e];
}

}  // namespace dbst
