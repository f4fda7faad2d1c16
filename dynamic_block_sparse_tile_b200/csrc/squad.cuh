// SQuad two-pass attention ("SQuad: Sub-Quadratic Attention Distillation for
// Efficient Video Generation", section "Methodology: SQuad", item
// "1. SQuad-Attention Operator").  A sequence of n = m * w tokens is split into
// m windows of w consecutive tokens.  The local pass attends within each window;
// the global pass attends across the tokens at the same offset of every window,
// with the local output as its values.
//
// Both passes are ordinary dense softmax attention on reshaped tensors, as the
// page's own design has it (standard attention blocks and tensor reshapes, no
// fused kernel): the local pass is the dense attention kernel on [B, H*m, w, D]
// (a free reshape), the global pass the same kernel on [B, H*w, m, D], which
// needs q, k and the local output with the two middle axes swapped.  This file
// holds that swap.
#pragma once
#include <cstdint>
#include "ptx.cuh"
#include "reorder.cuh"

namespace dbst {

// dst[head][r][a] = src[head][a][r] for rows of D bf16 (2^CPR_LOG2 16-byte chunks): token
// a*R + r of a head moves to row r*A + a.  HBM-bound permutation; consecutive threads write
// consecutive chunks of dst, and each thread issues kPermuteUnroll loads before its stores.
template <int CPR_LOG2>
__global__ void __launch_bounds__(256) window_transpose_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                               int A, int R, long long total) {
  constexpr int CPR = 1 << CPR_LOG2;
  const long long per_head = static_cast<long long>(A) * R;
  const long long step = static_cast<long long>(gridDim.x) * 256 * kPermuteUnroll;
  for (long long c0 = static_cast<long long>(blockIdx.x) * 256 * kPermuteUnroll + threadIdx.x; c0 < total;
       c0 += step) {
    uint4 v[kPermuteUnroll];
    long long d[kPermuteUnroll];
#pragma unroll
    for (int e = 0; e < kPermuteUnroll; ++e) {
      const long long c = c0 + 256LL * e;
      d[e] = -1;
      if (c < total) {
        const long long row = c >> CPR_LOG2;          // destination row
        const int ch = static_cast<int>(c & (CPR - 1));
        const long long head = row / per_head;
        const long long rem = row - head * per_head;
        const long long r = rem / A, a = rem - r * A;
        const long long srow = head * per_head + a * R + r;
        v[e] = ld_stream(src + (srow << CPR_LOG2) + ch);
        d[e] = c;
      }
    }
#pragma unroll
    for (int e = 0; e < kPermuteUnroll; ++e)
      if (d[e] >= 0) dst[d[e]] = v[e];
  }
}

}  // namespace dbst
