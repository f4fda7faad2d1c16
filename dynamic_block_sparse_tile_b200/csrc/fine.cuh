// Fine-grained key selection: key groups of 4 tokens (page "AB-Attention
// accélère la génération vidéo jusqu'à 2,23× en sautant 92% de l'attention",
// section "Les trois techniques", third technique: key/value blocks of only 4
// tokens).  Scoring and selection follow the NABLA path with the finer key unit:
// every 64-token query block is mean-pooled, every run of G = 4 consecutive
// tile-ordered key tokens ("group") is mean-pooled, the pooled logits are
// soft-maxed over all N/4 groups of the row, and the row keeps the smallest
// descending prefix of groups whose mass reaches p (ties to the lower group).
//
// Kernels:
//   group_pool_kernel<D, RASTER, G>  float64 means of G consecutive tile-ordered rows
//   fine_logits_kernel<D>            S[bh][i][g] = scale * <qp_i, kp_g> in float64
//   fine_select_kernel               one CTA per row: the CDF selection by a radix select on
//                                    64-bit keys, then the row's per-key-block group masks
// The selection's output is, per (b, h, query block i, key block j), a 16-bit mask of the
// kept groups of block j (bit r = tokens 4r .. 4r+3 of the block), and the ascending list of
// the key blocks with any kept group; the attention (sweep_kernel, offset mode) runs over
// those blocks and masks the other groups' columns.
#pragma once
#include <cstdint>
#include "ptx.cuh"
#include "reorder.cuh"

namespace dbst {

// out[r][:] = mean of rows G*r .. G*r+G-1 (tile order) of x, float64, for r < nrows_out.  One
// warp per output row; RASTER: x is in raster order and tile-ordered row t is read from its
// raster position.  G divides 64, so a group never leaves its tile.
template <int D, bool RASTER, int G>
__global__ void __launch_bounds__(256) group_pool_kernel(const uint4* __restrict__ x, double* __restrict__ out,
                                                         long long nrows_out, TileGeo tg) {
  static_assert(64 % G == 0, "groups stay inside a tile");
  constexpr int CPR = D / 8;            // 16-byte chunks per token row
  constexpr int RPW = 32 / CPR;         // token rows covered by one warp pass
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int ch = lane % CPR;
  const int r0 = lane / CPR;
  __shared__ int row_off[64];           // raster offset of tile row r from the tile's first token
  if (RASTER) {
    if (threadIdx.x < 64) row_off[threadIdx.x] = tiled_to_raster(threadIdx.x, tg);
    __syncthreads();
  }
  const long long per_head = tg.N / G;
  for (long long w = warp; w < nrows_out; w += nwarps) {
    const long long head = w / per_head;
    const int t0 = static_cast<int>(w - head * per_head) * G;   // first tile-ordered row of the group
    const int blk = t0 >> 6, rin = t0 & 63;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    for (int r = r0; r < G; r += RPW) {
      long long row;
      if constexpr (RASTER) row = head * tg.N + tiled_to_raster(blk * 64, tg) + row_off[rin + r];
      else row = head * tg.N + t0 + r;
      const uint4 v = ld_stream(x + row * CPR + ch);
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
      double* o = out + w * D + ch * 8;
#pragma unroll
      for (int e = 0; e < 8; e += 2)
        reinterpret_cast<double2*>(o)[e / 2] = make_double2(acc[e] / G, acc[e + 1] / G);
    }
  }
}

// S[bh][i][g] = scale * <qp[bh][i], kp[bh][g]>, float64; NQ query blocks by NK key groups per
// head.  64 x 64 outputs per CTA, 256 threads, 4 x 4 outputs per thread.
template <int D>
__global__ void __launch_bounds__(256) fine_logits_kernel(const double* __restrict__ qp,
                                                          const double* __restrict__ kp,
                                                          double* __restrict__ S, int NQ, int NK, double scale) {
  constexpr int KC = 16;
  __shared__ double As[KC][64 + 1];
  __shared__ double Bs[KC][64 + 1];
  const long long bh = blockIdx.z;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const double* Q = qp + bh * NQ * D;
  const double* K = kp + bh * NK * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
  for (int c0 = 0; c0 < D; c0 += KC) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = threadIdx.x + e * 256;
      const int row = idx / KC, col = idx % KC;
      As[col][row] = (i0 + row < NQ) ? Q[static_cast<long long>(i0 + row) * D + c0 + col] : 0.0;
      Bs[col][row] = (j0 + row < NK) ? K[static_cast<long long>(j0 + row) * D + c0 + col] : 0.0;
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
  double* out = S + bh * NQ * static_cast<long long>(NK);
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = i0 + ty + 16 * x;
    if (i >= NQ) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = j0 + tx + 16 * y;
      if (j < NK) out[static_cast<long long>(i) * NK + j] = acc[x][y] * scale;
    }
  }
}

constexpr int kFineThreads = 512;
constexpr int kFineMaxGroups = 16384;                  // NB <= 1024 blocks of 16 groups
constexpr int kFinePerThread = kFineMaxGroups / kFineThreads;
constexpr double kFineMassScale = 1099511627776.0;     // 2^40: masses as exact integer sums

// Key of group g with logit s: the order-preserving pattern of s in the top 48 bits, then
// 0xFFFF - g, so that a larger key is a larger logit, ties going to the lower group.
__device__ __forceinline__ uint64_t fine_key(double s, int g) {
  uint64_t u = static_cast<uint64_t>(__double_as_longlong(s));
  u = (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
  return (u & 0xFFFFFFFFFFFF0000ull) | static_cast<uint64_t>(0xFFFF - g);
}

// One CTA per row (b, h, i) of S [rows][NG] (NG = 16 * NB <= kFineMaxGroups).  Masses
// m_g = exp(s_g - max) are held as integers round(m_g * 2^40), so every sum below is exact and
// the selection does not depend on the order of the atomics.  With p >= 1 every group is kept.
// Radix select from the top 8 bits of the keys: each pass histograms the masses of the keys that
// share the prefix chosen so far into 256 buckets and picks, from the top, the bucket where the
// mass above plus the bucket's own reaches p * total.  After 8 passes (or once a bucket holds a
// single key) the prefix is the smallest kept key; every key at or above it is kept.
// Outputs: gmask[row][j] (bit r: group 16j + r kept), count[row] = key blocks with a kept group,
// idx[row][..] those blocks ascending.
__global__ void __launch_bounds__(kFineThreads) fine_select_kernel(const double* __restrict__ S, int NB, double p,
                                                                   uint16_t* __restrict__ gmask,
                                                                   int32_t* __restrict__ count,
                                                                   int16_t* __restrict__ idx) {
  __shared__ double s_red[kFineThreads / 32];
  __shared__ unsigned long long s_hist[256];
  __shared__ unsigned int s_cnt[256];
  __shared__ unsigned long long s_sel[4];   // prefix, mass above, bucket count, target
  __shared__ int s_wsum[kFineThreads / 32 + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NG = NB * 16;
  const long long row = blockIdx.x;
  const double* srow = S + row * NG;
  // row max
  double mx = -INFINITY;
  for (int g = tid; g < NG; g += kFineThreads) mx = fmax(mx, srow[g]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  if (warp == 0) {
    double v = lane < kFineThreads / 32 ? s_red[lane] : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == 0) s_red[0] = v;
  }
  __syncthreads();
  mx = s_red[0];
  // integer masses of this thread's groups g = tid + 512 e
  unsigned long long m[kFinePerThread];
  unsigned long long tot = 0;
#pragma unroll
  for (int e = 0; e < kFinePerThread; ++e) {
    const int g = tid + kFineThreads * e;
    m[e] = g < NG ? static_cast<unsigned long long>(llrint(exp(srow[g] - mx) * kFineMassScale)) : 0ull;
    tot += m[e];
  }
  if (tid < 256) {
    s_hist[tid] = 0ull;
    s_cnt[tid] = 0u;
  }
  if (tid == 0) {
    s_sel[0] = 0ull;
    s_sel[1] = 0ull;
    s_sel[2] = 0ull;
  }
  __syncthreads();
  atomicAdd(&s_hist[0], tot);               // the row total, in bucket 0 for one moment
  __syncthreads();
  const unsigned long long total = s_hist[0];
  __syncthreads();
  if (tid == 0) {
    s_hist[0] = 0ull;
    // target = ceil(p * total): the kept mass must reach p of the total
    const double t = p * static_cast<double>(total);
    s_sel[3] = (p >= 1.0) ? total : static_cast<unsigned long long>(ceil(t));
  }
  __syncthreads();
  uint64_t thr = 0;                         // smallest kept key (0 keeps everything)
  if (p < 1.0) {
    uint64_t prefix = 0, pmask = 0;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
#pragma unroll 4
      for (int e = 0; e < kFinePerThread; ++e) {
        const int g = tid + kFineThreads * e;
        if (g >= NG) break;
        const uint64_t key = fine_key(srow[g], g);
        if ((key & pmask) == prefix) {
          const int b = static_cast<int>((key >> shift) & 0xFF);
          atomicAdd(&s_hist[b], m[e]);
          atomicAdd(&s_cnt[b], 1u);
        }
      }
      __syncthreads();
      if (warp == 0) {
        // buckets from the top: lane l holds buckets 255 - 8l .. 248 - 8l
        unsigned long long hb[8], run = 0;
        unsigned int cb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          hb[u] = s_hist[255 - 8 * lane - u];
          cb[u] = s_cnt[255 - 8 * lane - u];
          run += hb[u];
        }
        unsigned long long incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const unsigned long long o = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += o;
        }
        const unsigned long long above0 = s_sel[1];
        const unsigned long long target = s_sel[3];
        unsigned long long acc = above0 + incl - run;   // mass above this lane's first bucket
        int found = -1;
        unsigned long long above_b = 0;
        unsigned int cnt_b = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (found < 0 && cb[u] > 0 && acc + hb[u] >= target) {
            found = 255 - 8 * lane - u;
            above_b = acc;
            cnt_b = cb[u];
          }
          acc += hb[u];
        }
        // the first lane (highest buckets) that found one decides; if none did (rounding), the
        // lowest non-empty bucket keeps everything that is left
        const unsigned int hit = __ballot_sync(0xffffffffu, found >= 0);
        int lowest = -1;
        unsigned long long above_low = 0;
        unsigned int cnt_low = 0;
        {
          unsigned long long a2 = above0 + incl - run;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (cb[u] > 0) {
              lowest = 255 - 8 * lane - u;
              above_low = a2;
              cnt_low = cb[u];
            }
            a2 += hb[u];
          }
        }
        const unsigned int nonempty = __ballot_sync(0xffffffffu, lowest >= 0);
        const int src = hit ? (__ffs(hit) - 1) : (31 - __clz(nonempty));
        const int fb = __shfl_sync(0xffffffffu, hit ? found : lowest, src);
        const unsigned long long fa = __shfl_sync(0xffffffffu, hit ? above_b : above_low, src);
        const unsigned int fc = __shfl_sync(0xffffffffu, hit ? cnt_b : cnt_low, src);
        if (lane == 0) {
          s_sel[0] = prefix | (static_cast<uint64_t>(fb) << shift);
          s_sel[1] = fa;
          s_sel[2] = fc;
        }
      }
      __syncthreads();
      prefix = s_sel[0];
      pmask |= 0xFFull << shift;
      const unsigned int nb = static_cast<unsigned int>(s_sel[2]);
      if (tid < 256) {
        s_hist[tid] = 0ull;
        s_cnt[tid] = 0u;
      }
      __syncthreads();
      if (nb == 1u) {   // one key left with this prefix: it is the threshold
        for (int e = 0; e < kFinePerThread; ++e) {
          const int g = tid + kFineThreads * e;
          if (g >= NG) break;
          const uint64_t key = fine_key(srow[g], g);
          if ((key & pmask) == prefix) s_sel[0] = key;   // exactly one thread writes
        }
        __syncthreads();
        prefix = s_sel[0];
        break;
      }
    }
    thr = prefix;
  }
  // group masks per key block (16 groups each), then the ascending list of blocks with any
  uint16_t* gm = gmask + row * NB;
  for (int j = tid; j < NB; j += kFineThreads) {
    uint32_t bitsj = 0u;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int g = 16 * j + r;
      if (fine_key(srow[g], g) >= thr) bitsj |= 1u << r;
    }
    gm[j] = static_cast<uint16_t>(bitsj);
  }
  // ascending list: one round of 512 blocks at a time, positions from a block-wide ballot scan
  __syncthreads();
  int base = 0;
  for (int j0 = 0; j0 < NB; j0 += kFineThreads) {
    const int j = j0 + tid;
    const bool has = j < NB && gm[j] != 0;
    const unsigned int bal = __ballot_sync(0xffffffffu, has);
    if (lane == 0) s_wsum[warp] = __popc(bal);
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int w = 0; w < kFineThreads / 32; ++w) {
        const int c = s_wsum[w];
        s_wsum[w] = run;
        run += c;
      }
      s_wsum[kFineThreads / 32] = run;
    }
    __syncthreads();
    if (has) idx[row * NB + base + s_wsum[warp] + __popc(bal & ((1u << lane) - 1u))] = static_cast<int16_t>(j);
    base += s_wsum[kFineThreads / 32];
    __syncthreads();
  }
  if (tid == 0) count[row] = base;
}

}  // namespace dbst
