// Sampled key-block selection with inclusion-probability weights: SIP on the
// page "AB-Attention accélère la génération vidéo jusqu'à 2,23× en sautant 92%
// de l'attention", section "Les trois techniques", second technique.  Blocks
// enter the sample with probability proportional to their score, the top ones
// with certainty, and each kept block carries the logit offset log(1/pi) that
// makes the softmax numerator and normaliser unbiased (Horvitz-Thompson).
//
// One warp per query-block row of the float64 pooled logits s_ij that the mask
// builder computes (the scores are the pooled map a = softmax_j(s_ij)):
//   pi_j  = min(1, c a_j) with sum_j pi_j = K: blocks with c a_j >= 1 are fixed
//           at 1 and c is recomputed over the rest until no block joins them
//           (all blocks with a_j > 0 get pi = 1 when K covers them all)
//   keep  = u_ij < pi_j for the caller's uniforms u (float64)
//   offset_ij = log(1 / pi_j) (float32) for kept blocks, 0 elsewhere
// and the same bitmask and ascending lists as the CDF selection.  Rows longer
// than 32 blocks are walked in strides of 32; the row's map a_j (one exponential
// per block) and its certainty flags (one bit per block) live in shared memory
// (kSipWarps * NB doubles of dynamic shared memory), so the fixed-point rounds
// only read them.
#pragma once
#include <cstdint>
#include "mask.cuh"
#include "ptx.cuh"

namespace dbst {

constexpr int kSipWarps = 4;           // warps (rows in flight) per CTA
constexpr int kSipMaxWords = 128;      // NB <= 4096

__device__ __forceinline__ int warp_sum_i32(int v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__global__ void __launch_bounds__(32 * kSipWarps) sip_select_kernel(const double* __restrict__ S, int NB, int NW,
                                                                    long long rows, double K,
                                                                    const double* __restrict__ u,
                                                                    uint32_t* __restrict__ bits,
                                                                    int32_t* __restrict__ count,
                                                                    int16_t* __restrict__ idx,
                                                                    float* __restrict__ offsets) {
  __shared__ uint32_t s_cert[kSipWarps][kSipMaxWords];
  extern __shared__ double s_a[];              // [kSipWarps][NB]
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint32_t* cert = s_cert[wib];
  double* arow = s_a + static_cast<long long>(wib) * NB;
  const long long warp0 = static_cast<long long>(blockIdx.x) * kSipWarps + wib;
  const long long nwarps = static_cast<long long>(gridDim.x) * kSipWarps;
  for (long long row = warp0; row < rows; row += nwarps) {
    const double* srow = S + row * NB;
    const double* urow = u + row * NB;
    // pooled map a_j = exp(s_j - max) / sum
    double mx = -INFINITY;
    for (int j = lane; j < NB; j += 32) mx = fmax(mx, srow[j]);
    mx = warp_max_f64(mx);
    double sum = 0.0;
    for (int j = lane; j < NB; j += 32) {
      const double e = exp(srow[j] - mx);
      arow[j] = e;
      sum += e;
    }
    sum = warp_sum_f64(sum);
    for (int j = lane; j < NB; j += 32) arow[j] /= sum;   // each lane rereads only its own entries
    auto a_of = [&](int j) -> double { return arow[j]; };
    int npos = 0;
    for (int j = lane; j < NB; j += 32) npos += a_of(j) > 0.0;
    npos = warp_sum_i32(npos);
    for (int w = lane; w < NW; w += 32) cert[w] = 0u;
    __syncwarp();
    const bool all = K >= static_cast<double>(npos);
    double c = 0.0;
    if (!all) {
      for (int it = 0; it <= NB; ++it) {   // each round fixes at least one more block, or stops
        double rest = 0.0;
        int ncert = 0;
        for (int j = lane; j < NB; j += 32) {
          const bool cj = (cert[j >> 5] >> (j & 31)) & 1u;
          ncert += cj;
          if (!cj) {
            const double a = a_of(j);
            if (a > 0.0) rest += a;
          }
        }
        rest = warp_sum_f64(rest);
        ncert = warp_sum_i32(ncert);
        c = (K - static_cast<double>(ncert)) / rest;
        int nnew = 0;
        for (int j0 = 0; j0 < NB; j0 += 32) {
          const int j = j0 + lane;
          bool add = false;
          if (j < NB && !((cert[j >> 5] >> (j & 31)) & 1u)) {
            const double a = a_of(j);
            add = a > 0.0 && c * a >= 1.0;
          }
          const uint32_t m = __ballot_sync(0xffffffffu, add);
          if (lane == 0) cert[j0 >> 5] |= m;
          nnew += __popc(m);
        }
        __syncwarp();
        if (nnew == 0) break;
      }
    }
    // sample, offsets, bitmask and lists
    int base = 0;
    for (int j0 = 0; j0 < NB; j0 += 32) {
      const int j = j0 + lane;
      bool keep = false;
      float off = 0.0f;
      if (j < NB) {
        const double a = a_of(j);
        double pi = 0.0;
        if (a > 0.0) pi = (all || ((cert[j >> 5] >> (j & 31)) & 1u)) ? 1.0 : c * a;
        keep = urow[j] < pi;
        if (keep) off = static_cast<float>(-log(pi));
        offsets[row * NB + j] = off;
      }
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) bits[row * NW + (j0 >> 5)] = m;
      if (keep) idx[row * NB + base + __popc(m & ((1u << lane) - 1u))] = static_cast<int16_t>(j);
      base += __popc(m);
    }
    if (lane == 0) count[row] = base;
    __syncwarp();   // the next row overwrites cert and arow
  }
}

}  // namespace dbst
