// Query-block pairing for the query-pair attention kernel.
//
// The attention kernel runs two 64-token query blocks per CTA over the union of
// their kept key-block lists, so a pair costs ceil(|A u B| / 2) tiles of two key
// blocks.  Pairing blocks whose lists overlap saves tensor-core work; the kept
// sets themselves (the NABLA page's mask) are untouched, only the schedule
// changes.
//
// One CTA per (b, h).  Candidate partners are the six face neighbours of a block
// on the tile grid (+-1 along t, y and x), where content-adaptive lists overlap
// most.  An edge (v, u) weighs the tiles the pair saves over running v and u
// alone:  ceil(|A|/2) + ceil(|B|/2) - ceil(|A u B|/2), which is never negative.
// The matching takes locally dominant edges in rounds: an unmatched block points
// at its heaviest unmatched neighbour (ties to the lower index) and mutual
// pointers are matched.  Every round matches at least one edge while candidate
// edges remain (the lowest-indexed block that has an edge of the largest
// remaining weight and its lowest-indexed such neighbour point at each other).
// Blocks left unmatched are then paired in ascending order (never worse than
// running them alone), with one single block when their count is odd.
//
// Output pairs[bh][e], e < ceil(NB/2): qa | qb << 16, qb = 0xFFFF for a single
// block, longest first: by the pair's tiles ceil(|A u B| / 2) descending, ties
// by the order of construction (matched pairs by lower block index, then the
// leftover pairs).  The attention kernel starts the longest items first.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace dbst {

constexpr int kPairingThreads = 512;
// A head's mask rows are staged in shared memory when they fit in this many bytes.
constexpr int kPairingStageBytes = 96 * 1024;
constexpr int kPairingMaxRounds = 64;

struct PairingGeo {
  int NB, NW;            // blocks per head, mask words per row
  int nX, nY, nT;        // tile grid
};

__device__ __forceinline__ int pairing_neighbour(int v, int k, const PairingGeo& g) {
  const int x = v % g.nX, y = (v / g.nX) % g.nY, t = v / (g.nX * g.nY);
  switch (k) {
    case 0: return x > 0 ? v - 1 : -1;
    case 1: return x + 1 < g.nX ? v + 1 : -1;
    case 2: return y > 0 ? v - g.nX : -1;
    case 3: return y + 1 < g.nY ? v + g.nX : -1;
    case 4: return t > 0 ? v - g.nX * g.nY : -1;
    default: return t + 1 < g.nT ? v + g.nX * g.nY : -1;
  }
}

// Block-wide exclusive scan of one int per thread (kPairingThreads / 32 <= 32 warps); the total
// goes to *total.
__device__ __forceinline__ int pairing_scan(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kPairingThreads / 32 ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < kPairingThreads / 32) warp_sums[lane] = wi - w;
    if (lane == kPairingThreads / 32 - 1) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  __syncthreads();
  return r;
}

// Dynamic shared memory: count[NB], weight[NB][6], partner[NB], best[NB] (ints), scan scratch,
// then (STAGE) the head's mask rows.
template <bool STAGE>
__global__ void __launch_bounds__(kPairingThreads) pair_blocks_kernel(const uint32_t* __restrict__ bits, PairingGeo g,
                                                                      int32_t* __restrict__ pairs) {
  extern __shared__ int pairing_smem[];
  const int NB = g.NB;
  int* count = pairing_smem;
  int* weight = count + NB;
  int* partner = weight + 6 * NB;
  int* best = partner + NB;
  int* scratch = best + NB;              // 16 warp sums + 2 totals + change flag
  volatile int* changed = scratch + 18;
  const long long bh = blockIdx.x;
  const uint32_t* gh = bits + bh * static_cast<long long>(NB) * g.NW;
  const int tid = threadIdx.x;
  const uint32_t* head = gh;
  if constexpr (STAGE) {
    uint32_t* st = reinterpret_cast<uint32_t*>(scratch + 32);
    for (int i = tid; i < NB * g.NW; i += kPairingThreads) st[i] = gh[i];
    head = st;
    __syncthreads();
  }

  // Rows in shared memory: one thread per block.  Rows in global memory (a head too large to stage):
  // one warp per block, the lanes holding the row's words w = lane + 32 i (NW <= 128), so that every
  // read of a row is one coalesced pass.  First the kept counts and each neighbour's union count,
  // then the weights.
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int kWarps = kPairingThreads / 32;
  if constexpr (STAGE) {
    for (int v = tid; v < NB; v += kPairingThreads) {
      int c = 0;
      for (int w = 0; w < g.NW; ++w) c += __popc(head[static_cast<long long>(v) * g.NW + w]);
      count[v] = c;
      partner[v] = -1;
    }
    __syncthreads();
    for (int v = tid; v < NB; v += kPairingThreads) {
      const uint32_t* a = head + static_cast<long long>(v) * g.NW;
      for (int k = 0; k < 6; ++k) {
        const int u = pairing_neighbour(v, k, g);
        int un = -1;
        if (u >= 0) {
          const uint32_t* b = head + static_cast<long long>(u) * g.NW;
          un = 0;
          for (int w = 0; w < g.NW; ++w) un += __popc(a[w] | b[w]);
        }
        weight[v * 6 + k] = un;   // union count for now; -1: no neighbour
      }
    }
  } else for (int v = warp; v < NB; v += kWarps) {
    const uint32_t* a = head + static_cast<long long>(v) * g.NW;
    uint32_t aw[4];
    int c = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int w = lane + 32 * i;
      aw[i] = w < g.NW ? a[w] : 0u;
      c += __popc(aw[i]);
    }
    c = __reduce_add_sync(0xffffffffu, c);
    int un[6];
#pragma unroll
    for (int k = 0; k < 6; ++k) {
      const int u = pairing_neighbour(v, k, g);
      int x = 0;
      if (u >= 0) {
        const uint32_t* b = head + static_cast<long long>(u) * g.NW;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int w = lane + 32 * i;
          x += __popc(aw[i] | (w < g.NW ? b[w] : 0u));
        }
      }
      un[k] = u >= 0 ? x : -1;
    }
#pragma unroll
    for (int k = 0; k < 6; ++k) {
      const int x = un[k] >= 0 ? __reduce_add_sync(0xffffffffu, un[k]) : -1;
      if (lane == 0) weight[v * 6 + k] = x;   // union count for now; -1: no neighbour
    }
    if (lane == 0) {
      count[v] = c;
      partner[v] = -1;
    }
  }
  __syncthreads();
  for (int v = tid; v < NB; v += kPairingThreads) {
    for (int k = 0; k < 6; ++k) {
      const int u = pairing_neighbour(v, k, g);
      const int x = weight[v * 6 + k];
      weight[v * 6 + k] = u >= 0 ? (count[v] + 1) / 2 + (count[u] + 1) / 2 - (x + 1) / 2 : -1;
    }
  }
  __syncthreads();

  // locally dominant matching over the candidate edges
  for (int round = 0; round < kPairingMaxRounds; ++round) {
    for (int v = tid; v < NB; v += kPairingThreads) {
      int bu = -1, bw = -1;
      if (partner[v] < 0) {
        for (int k = 0; k < 6; ++k) {
          const int u = pairing_neighbour(v, k, g);
          if (u < 0 || partner[u] >= 0) continue;
          const int wt = weight[v * 6 + k];
          if (wt > bw || (wt == bw && u < bu)) {
            bw = wt;
            bu = u;
          }
        }
      }
      best[v] = bu;
    }
    if (tid == 0) *changed = 0;
    __syncthreads();
    for (int v = tid; v < NB; v += kPairingThreads) {
      const int u = best[v];
      if (u >= 0 && v < u && best[u] == v) {
        partner[v] = u;
        partner[u] = v;
        *changed = 1;
      }
    }
    __syncthreads();
    const bool more = *changed != 0;
    __syncthreads();
    if (!more) break;
  }

  // output: matched pairs (by lower index), then the leftovers paired in ascending order
  constexpr int PER = 4096 / kPairingThreads;   // blocks per thread in the scans (NB <= 4096)
  const int v0 = tid * PER;
  int leads = 0, lefts = 0;
  for (int i = 0; i < PER; ++i) {
    const int v = v0 + i;
    if (v >= NB) break;
    leads += (partner[v] > v);
    lefts += (partner[v] < 0);
  }
  const int lead_base = pairing_scan(leads, scratch, scratch + 16);
  const int n_lead = scratch[16];
  const int left_base = pairing_scan(lefts, scratch, scratch + 17);
  const int n_left = scratch[17];
  int32_t* out = pairs + bh * ((NB + 1) / 2);
  int li = lead_base, fi = left_base;
  for (int i = 0; i < PER; ++i) {
    const int v = v0 + i;
    if (v >= NB) break;
    if (partner[v] > v) out[li++] = static_cast<int32_t>(static_cast<uint32_t>(v) | (static_cast<uint32_t>(partner[v]) << 16));
    if (partner[v] < 0) {
      // leftover number fi: the even ones start a pair with the next leftover
      if ((fi & 1) == 0) {
        // find the next leftover (fi + 1) by scanning forward; leftovers are sparse
        int w = -1;
        if (fi + 1 < n_left)
          for (int u = v + 1; u < NB; ++u)
            if (partner[u] < 0) {
              w = u;
              break;
            }
        out[n_lead + fi / 2] = static_cast<int32_t>(static_cast<uint32_t>(v) | (static_cast<uint32_t>(w >= 0 ? w : 0xFFFF) << 16));
      }
      ++fi;
    }
  }
  __syncthreads();

  // longest first: each pair's tiles, then its rank (tiles descending, construction order on ties)
  const int npairs = (NB + 1) / 2;
  int* ent = weight;              // the edge weights are no longer needed: 6 NB >= 2 npairs ints
  int* cost = weight + npairs;
  for (int e = STAGE ? tid : warp; e < npairs; e += STAGE ? kPairingThreads : kWarps) {
    const int32_t x = out[e];
    const int a = x & 0xFFFF, b = (x >> 16) & 0xFFFF;
    int un = 0;
    if (b == 0xFFFF) {
      un = count[a];
    } else if (STAGE) {
      const uint32_t* ra = head + static_cast<long long>(a) * g.NW;
      const uint32_t* rb = head + static_cast<long long>(b) * g.NW;
      for (int w = 0; w < g.NW; ++w) un += __popc(ra[w] | rb[w]);
    } else {   // one warp per pair, coalesced rows
      const uint32_t* ra = head + static_cast<long long>(a) * g.NW;
      const uint32_t* rb = head + static_cast<long long>(b) * g.NW;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int w = lane + 32 * i;
        un += w < g.NW ? __popc(ra[w] | rb[w]) : 0;
      }
      un = __reduce_add_sync(0xffffffffu, un);
    }
    if (STAGE || lane == 0) {
      ent[e] = x;
      cost[e] = (un + 1) / 2;
    }
  }
  __syncthreads();
  for (int e = tid; e < npairs; e += kPairingThreads) {
    const int c = cost[e];
    int rank = 0;
    for (int f = 0; f < npairs; ++f) {
      const int cf = cost[f];
      rank += (cf > c) || (cf == c && f < e);
    }
    out[rank] = ent[e];
  }
}

inline size_t pairing_rows_bytes(int NB, int NW) { return static_cast<size_t>(NB) * NW * sizeof(uint32_t); }
inline size_t pairing_smem_bytes(int NB, int NW, bool stage) {
  return static_cast<size_t>(NB) * 9 * sizeof(int) + 32 * sizeof(int) + (stage ? pairing_rows_bytes(NB, NW) : 0);
}

}  // namespace dbst
