// Adaptive block mask: block mean-pool, pooled score map, per-row CDF
// selection, sliding-tile union and index-list expansion (NABLA page,
// "Construction de Masque Adaptatif" and "Intégration Hybride avec STA").
//
// Precision: the pooled means are exact (64 bf16 values summed in float64) and
// the pooled logits are float64.  The order of a row's blocks comes from those
// logits, with float64 exponentials and sums for the masses; the kept set agrees
// with a float64 reference except where a cumulative mass sits within rounding
// of p.  Rows of at most 2048 blocks are built by the tensor-core path of
// mask_tc.cuh; these kernels serve longer rows, and the pool and logits serve the
// SIP mask.
#pragma once
#include <cstdint>
#include "ptx.cuh"
#include "reorder.cuh"

namespace dbst {

// ---------------------------------------------------------------------------
// Block mean-pool: one warp per 64-token block; out[blk][c] = mean (float64).
// RASTER: q and k are in raster token order and the block's rows are gathered
// through the tile permutation (the same rows, summed in the same order).  A
// row's raster offset from its tile's first token depends only on the row's
// place in the tile, so the 64 offsets are tabulated once per CTA.
// ---------------------------------------------------------------------------
template <int D, bool RASTER>
__global__ void __launch_bounds__(256) pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                   double* __restrict__ qp, double* __restrict__ kp,
                                                   long long nblocks, int NB, TileGeo tg) {
  constexpr int CPR = D / 8;            // 16-byte chunks per token row
  constexpr int RPW = 32 / CPR;         // token rows covered by one warp pass
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int ch = lane % CPR;
  const int r0 = lane / CPR;
  __shared__ int row_off[64];             // raster offset of tile row r from the tile's first token
  if (RASTER) {
    if (threadIdx.x < 64) row_off[threadIdx.x] = tiled_to_raster(threadIdx.x, tg);   // tile 0 starts at token 0
    __syncthreads();
  }
  for (long long w = warp; w < 2 * nblocks; w += nwarps) {
    const bool isk = w >= nblocks;
    const long long b = isk ? w - nblocks : w;
    const uint4* src = (isk ? k : q) + b * 64 * CPR;
    const int blk = static_cast<int>(b % NB);
    const uint4* head = (isk ? k : q) +
                        ((b / NB) * static_cast<long long>(tg.N) + (RASTER ? tiled_to_raster(blk * 64, tg) : 0)) * CPR;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 8
    for (int r = r0; r < 64; r += RPW) {
      const uint4 v = RASTER ? ld_stream(head + row_off[r] * CPR + ch) : ld_stream(src + r * CPR + ch);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += static_cast<double>(__uint_as_float(u[e] << 16));
        acc[2 * e + 1] += static_cast<double>(__uint_as_float(u[e] & 0xFFFF0000u));
      }
    }
#pragma unroll
    for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    if (r0 == 0) {
      double* out = (isk ? kp : qp) + b * D + ch * 8;
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        double2 pr = make_double2(acc[e] * (1.0 / 64.0), acc[e + 1] * (1.0 / 64.0));
        reinterpret_cast<double2*>(out)[e / 2] = pr;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Pooled logits S[bh][i][j] = scale * <Qp_i, Kp_j> in float64.
// 64 x 64 output tile per CTA, 256 threads, 4 x 4 outputs per thread.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pooled_logits_kernel(const double* __restrict__ qp,
                                                            const double* __restrict__ kp,
                                                            double* __restrict__ S, int NB, double scale) {
  constexpr int KC = 16;
  __shared__ double As[KC][64 + 1];
  __shared__ double Bs[KC][64 + 1];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const double* Q = qp + static_cast<long long>(bh) * NB * D;
  const double* K = kp + static_cast<long long>(bh) * NB * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
  for (int c0 = 0; c0 < D; c0 += KC) {
    // 64 rows x 16 columns of each operand: 1024 values, 4 per thread
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = threadIdx.x + e * 256;
      const int row = idx / KC, col = idx % KC;
      As[col][row] = (i0 + row < NB) ? Q[static_cast<long long>(i0 + row) * D + c0 + col] : 0.0;
      Bs[col][row] = (j0 + row < NB) ? K[static_cast<long long>(j0 + row) * D + c0 + col] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      double a[4], b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a[e] = As[c][ty + 16 * e];
        b[e] = Bs[c][tx + 16 * e];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fma(a[x], b[y], acc[x][y]);
    }
    __syncthreads();
  }
  double* out = S + static_cast<long long>(bh) * NB * NB;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = i0 + ty + 16 * x;
    if (i >= NB) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = j0 + tx + 16 * y;
      if (j < NB) out[static_cast<long long>(i) * NB + j] = acc[x][y] * scale;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-row softmax + CDF selection + STA union + list expansion.
// One CTA (256 threads) per row; thread t owns key blocks j = t + 256*u.
//
// Selection: every block gets a 64-bit key that orders the row by A
// descending with ties to the lower index,
//   key = [octave of A: 8 bits][top 40 mantissa bits of A][0xFFFF - j],
// the keys are sorted descending with a shared-memory bitonic network, the
// masses are prefix-summed in that order (float64), and the first position
// whose cumulative mass reaches p fixes the threshold key.  Values below
// 2^-255 share octave 0; they are never at the threshold for p < 1, since the
// mass above them exceeds 1 - NB * 2^-255.  Values equal in their top 40
// mantissa bits count as ties.
// ---------------------------------------------------------------------------
struct SelectGeo {
  int NB, NW;          // blocks per (b,h); 32-bit mask words per row
  int nX, nY;          // tile grid (for the sliding-tile neighbourhood)
  int sta_radius;      // < 0: none
  double p;            // CDF threshold; >= 1 keeps all
};

__device__ __forceinline__ double block_reduce_max(double v, double* red) {
  for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double r = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) r = fmax(r, red[i]);
  return r;
}
__device__ __forceinline__ double block_reduce_sum(double v, double* red) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double r = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) r += red[i];
  return r;
}

__device__ __forceinline__ double p_of(const SelectGeo& g) { return g.p; }

__device__ __forceinline__ unsigned long long select_key(double a, int j) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(a));
  const int e = static_cast<int>(b >> 52) - 768;                 // A in (0,1]: biased exponent <= 1023
  const unsigned long long oct = static_cast<unsigned long long>(e < 0 ? 0 : e);
  const unsigned long long man = (b & ((1ull << 52) - 1)) >> 12;  // top 40 mantissa bits
  return (oct << 56) | (man << 16) | static_cast<unsigned long long>(0xFFFF - j);
}

// dynamic shared memory: keys [256*NPT] u64, masses [256*NPT] f64
template <int NPT>
__global__ void __launch_bounds__(256) select_kernel(const double* __restrict__ S, SelectGeo g,
                                                     uint32_t* __restrict__ bits, int32_t* __restrict__ count,
                                                     int16_t* __restrict__ idx) {
  constexpr int NP2 = 256 * NPT;
  extern __shared__ __align__(16) unsigned char sel_smem[];
  unsigned long long* s_key = reinterpret_cast<unsigned long long*>(sel_smem);
  double* s_a = reinterpret_cast<double*>(sel_smem + NP2 * 8);
  __shared__ double red[8];
  __shared__ double wsum[8];
  __shared__ int s_first;
  __shared__ int wcount[128 + 1];

  const long long row = blockIdx.x;
  const int i = static_cast<int>(row % g.NB);
  const double* srow = S + row * g.NB;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  double a[NPT];
  unsigned long long key[NPT];
  double mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const int j = t + 256 * u;
    a[u] = (j < g.NB) ? srow[j] : -INFINITY;
    mx = fmax(mx, a[u]);
  }
  mx = block_reduce_max(mx, red);
  double sum = 0.0;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const int j = t + 256 * u;
    a[u] = (j < g.NB) ? exp(a[u] - mx) : 0.0;
    sum += a[u];
  }
  sum = block_reduce_sum(sum, red);
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const int j = t + 256 * u;
    a[u] = a[u] / sum;
    key[u] = (j < g.NB) ? select_key(a[u], j) : 0ull;
    s_key[j] = key[u];
    s_a[j] = a[u];
  }

  unsigned long long thr = 0ull;   // keep key >= thr (0 keeps all)
  if (g.p < 1.0) {
    __syncthreads();
    // bitonic sort, descending
    for (int k = 2; k <= NP2; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
#pragma unroll
        for (int e = 0; e < NPT / 2 + (NPT == 1); ++e) {
          const int pi = t + 256 * e;
          if (pi < NP2 / 2) {
            const int lo = 2 * pi - (pi & (jj - 1));
            const int hi = lo + jj;
            const unsigned long long x = s_key[lo], y = s_key[hi];
            const bool desc = (lo & k) == 0;
            if (desc ? (x < y) : (x > y)) {
              s_key[lo] = y;
              s_key[hi] = x;
            }
          }
        }
        __syncthreads();
      }
    }
    // masses in sorted order, prefix-summed: thread t owns sorted positions [t*NPT, (t+1)*NPT)
    double m[NPT];
    double local = 0.0;
#pragma unroll
    for (int u = 0; u < NPT; ++u) {
      const int r = t * NPT + u;
      m[u] = (r < g.NB) ? s_a[0xFFFF - static_cast<int>(s_key[r] & 0xFFFFull)] : 0.0;
      local += m[u];
    }
    double incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) wsum[warp] = incl;
    if (t == 0) s_first = 0x7FFFFFFF;
    __syncthreads();
    double before = incl - local;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    double c = before;
#pragma unroll
    for (int u = 0; u < NPT; ++u) {
      const int r = t * NPT + u;
      c += m[u];
      if (r < g.NB && c >= g.p) {
        atomicMin(&s_first, r);
        break;
      }
    }
    __syncthreads();
    const int first = s_first;
    thr = (first < g.NB) ? s_key[first] : 0ull;   // no crossing (rounding): keep every block
  }

  // tile coordinates of the query block (for the sliding-tile neighbourhood)
  const int qx = i % g.nX, qy = (i / g.nX) % g.nY, qt = i / (g.nX * g.nY);
  uint32_t words[NPT];
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const int j = t + 256 * u;
    bool keep = false;
    if (j < g.NB) {
      keep = key[u] >= thr;
      if (g.sta_radius >= 0) {
        const int kx = j % g.nX, ky = (j / g.nX) % g.nY, kt = j / (g.nX * g.nY);
        const int dmax = max(abs(kt - qt), max(abs(ky - qy), abs(kx - qx)));
        keep = keep || (dmax <= g.sta_radius);
      }
    }
    words[u] = __ballot_sync(0xffffffffu, keep);
  }
  // word index of (warp, u) is 8*u + warp; store words and per-word counts
  uint32_t* brow = bits + row * g.NW;
  if (lane == 0) {
#pragma unroll
    for (int u = 0; u < NPT; ++u) {
      const int w = 8 * u + warp;
      if (w < g.NW) {
        brow[w] = words[u];
        wcount[w] = __popc(words[u]);
      }
    }
  }
  __syncthreads();
  if (t == 0) {
    int run = 0;
    for (int w = 0; w < g.NW; ++w) {
      const int cw = wcount[w];
      wcount[w] = run;
      run += cw;
    }
    wcount[g.NW] = run;
    count[row] = run;
  }
  __syncthreads();
  int16_t* irow = idx + row * g.NB;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const int w = 8 * u + warp;
    if (w < g.NW && ((words[u] >> lane) & 1u)) {
      const int pos = wcount[w] + __popc(words[u] & ((1u << lane) - 1u));
      irow[pos] = static_cast<int16_t>(t + 256 * u);
    }
  }
}

// Warp reductions in float64 (the SIP selection and the tensor-core mask's band refinement).
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ double warp_max_f64(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// ---------------------------------------------------------------------------
// Caller-supplied bitmask -> counts + ascending index lists.  One warp per row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bits_to_lists_kernel(const uint32_t* __restrict__ bits, int NB, int NW,
                                                            long long rows, int32_t* __restrict__ count,
                                                            int16_t* __restrict__ idx) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long row = warp; row < rows; row += nwarps) {
    const uint32_t* brow = bits + row * NW;
    int16_t* irow = idx + row * NB;
    int base = 0;
    for (int w0 = 0; w0 < NW; w0 += 32) {
      const int w = w0 + lane;
      uint32_t word = (w < NW) ? brow[w] : 0u;
      if (w == NW - 1 && (NB & 31)) word &= (1u << (NB & 31)) - 1u;   // ignore bits past NB
      const int c = __popc(word);
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      int pos = base + incl - c;
      while (word) {
        const int b = __ffs(word) - 1;
        word &= word - 1u;
        irow[pos++] = static_cast<int16_t>(w * 32 + b);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) count[row] = base;
  }
}

}  // namespace dbst
