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

// to_tiled = 1: dst[tiled r] = src[raster n(r)];  0: dst[raster n(r)] = src[tiled r].
template <int CPR_LOG2>
__global__ void __launch_bounds__(256) tile_permute_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           TileGeo g, long long rows, int to_tiled) {
  constexpr int CPR = 1 << CPR_LOG2;   // 16-byte chunks per token row
  const long long total = rows << CPR_LOG2;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < total; c += stride) {
    const long long row = c >> CPR_LOG2;
    const int ch = static_cast<int>(c & (CPR - 1));
    const long long bh = row / g.N;
    const int r = static_cast<int>(row - bh * g.N);
    const int n = tiled_to_raster(r, g);
    const long long tiled_off = (row << CPR_LOG2) + ch;
    const long long raster_off = ((bh * g.N + n) << CPR_LOG2) + ch;
    if (to_tiled) {
      dst[tiled_off] = ld_stream(src + raster_off);
    } else {
      dst[raster_off] = ld_stream(src + tiled_off);
    }
  }
}

}  // namespace dbst
