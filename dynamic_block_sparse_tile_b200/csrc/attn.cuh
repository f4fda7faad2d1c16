// Block-sparse exact softmax attention on sm_100a tensor cores ("Expansion"
// step on the NABLA page: attention over the tokens of the kept 64 x 64 tile
// pairs only).
//
// Formulation ("key-major").  One CTA owns one 64-token query block and walks
// its list of kept key blocks two at a time:
//     S^T[128 keys x 64 queries] = K_tile[128 x D] . Q_blk[64 x D]^T   (tcgen05, M=128, N=64)
//     O^T[D x 64 queries]       += V_tile^T[D x 128] . P^T[128 x 64]    (tcgen05, M=128, N=64)
// M is always 128 *keys* taken from the list, so any two kept blocks fill a
// full-rate tile and no query rows are wasted, whatever the mask.  Softmax
// runs over keys, i.e. over TMEM lanes: each thread owns one key row of S^T
// and keeps per-query partial sums; the running max is a CTA-wide per-query
// reference, refreshed only when a tile exceeds it by more than kRescaleLog2
// (exact: numerator and denominator share the same reference).
//
// Warp roles (256 threads): warp 0 issues TMA loads, warp 1 issues MMAs
// (one thread), warp 2 owns the TMEM allocation, warps 4-7 run the softmax
// and the epilogue (warp 4+q owns TMEM lanes 32q..32q+31).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace dbst {

constexpr int kStages = 2;
constexpr float kRescaleLog2 = 16.0f;

struct AttnParams {
  const int32_t* kv_count;   // [BH*NB]; null => dense (every list is 0..NB-1)
  const int16_t* kv_idx;     // [BH*NB*NB]
  __nv_bfloat16* o;          // tiled [BH, N, D]
  float* lse;                // [BH, N] or null
  int NB, N;
  float scale_log2;          // softmax scale * log2(e)
};

// Shared-memory plan (byte offsets from a 1024-aligned base).
struct AttnSmem {
  static constexpr int kQ = 0;                          // Q: D/64 regions of [64 rows x 128 B]
  static constexpr int kK = kQ + 16384;                 // K stages: 2 D-halves x [128 keys x 128 B]
  static constexpr int kKStage = 32768;
  static constexpr int kV = kK + kStages * kKStage;     // V stages, same layout (D=64: half 1 = zeros)
  static constexpr int kP = kV + kStages * kKStage;     // P^T buffers: [128 keys x 64 queries] bf16
  static constexpr int kPBuf = 16384;
  static constexpr int kList = kP + 2 * kPBuf;          // compacted key-block list, int16 x 4096
  static constexpr int kRed = kList + 8192;             // float [4][64] column max exchange
  static constexpr int kLsum = kRed + 1024;             // float [4][64] column sums
  static constexpr int kFinal = kLsum + 1024;           // float [2][64] final max / sum
  static constexpr int kBars = kFinal + 512;            // mbarriers
  static constexpr int kMisc = kBars + 256;             // tmem base, counts, abort flag
  static constexpr int kBytes = kMisc + 64;
};

// barrier slots (8 bytes each)
enum {
  BAR_Q = 0,
  BAR_KFULL = 1,                  // + stage
  BAR_VFULL = BAR_KFULL + kStages,
  BAR_KVEMPTY = BAR_VFULL + kStages,
  BAR_SFULL = BAR_KVEMPTY + kStages,  // + 2
  BAR_SEMPTY = BAR_SFULL + 2,
  BAR_PFULL = BAR_SEMPTY + 2,
  BAR_PEMPTY = BAR_PFULL + 2,
  BAR_OFULL = BAR_PEMPTY + 2,
  BAR_DRAIN = BAR_OFULL + 1,
  BAR_COUNT = BAR_DRAIN + 1
};

__device__ __forceinline__ bool bar_red_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int DH = D / 64;                 // 128-byte column halves per token row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  int16_t* s_list = reinterpret_cast<int16_t*>(sm + AttnSmem::kList);
  float* s_red = reinterpret_cast<float*>(sm + AttnSmem::kRed);
  float* s_lsum = reinterpret_cast<float*>(sm + AttnSmem::kLsum);
  float* s_final = reinterpret_cast<float*>(sm + AttnSmem::kFinal);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(sm + AttnSmem::kMisc);
  volatile uint32_t* s_abort = s_misc + 2;
  auto bar = [&](int slot) -> uint32_t { return sbase + AttnSmem::kBars + 8u * slot; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NB = prm.NB;
  const long long bh = blockIdx.x / NB;
  const int qb = blockIdx.x - static_cast<int>(bh * NB);
  const long long row0 = bh * prm.N + static_cast<long long>(qb) * 64;   // first query token row

  // ---- list of kept key blocks -> shared memory (drop out-of-range entries)
  int n_raw;
  const int16_t* gl = nullptr;
  if (prm.kv_count == nullptr) {
    n_raw = NB;
  } else {
    n_raw = prm.kv_count[bh * NB + qb];
    gl = prm.kv_idx + (bh * NB + qb) * static_cast<long long>(NB);
    if (n_raw < 0 || n_raw > NB) {
      if (tid == 0) record_error(kErrBounds);
      n_raw = n_raw < 0 ? 0 : NB;
    }
  }
  if (tid == 0) {
    for (int b = 0; b < BAR_COUNT; ++b) {
      uint32_t cnt = 1;
      if (b == BAR_SEMPTY || b == BAR_SEMPTY + 1 || b == BAR_PFULL || b == BAR_PFULL + 1) cnt = 128;
      mbar_init(bar(b), cnt);
    }
    fence_mbar_init();
    s_misc[1] = 0;
    s_misc[2] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n_raw; base += 256) {
    const int e = base + tid;
    int j = -1;
    if (e < n_raw) j = gl ? static_cast<int>(gl[e]) : e;
    const bool ok = (e < n_raw) && j >= 0 && j < NB;
    if (e < n_raw && !ok) record_error(kErrBounds);
    const unsigned ball = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) s_red[warp] = __int_as_float(__popc(ball));
    __syncthreads();
    int before = static_cast<int>(s_misc[1]);
    for (int w = 0; w < warp; ++w) before += __float_as_int(s_red[w]);
    if (ok) s_list[before + __popc(ball & ((1u << lane) - 1u))] = static_cast<int16_t>(j);
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < 8; ++w) tot += __float_as_int(s_red[w]);
      s_misc[1] += tot;
    }
    __syncthreads();
  }
  const int n = static_cast<int>(s_misc[1]);

  if (n == 0) {   // no kept key block: o = 0, lse = -inf
    const int chunks = 64 * D / 8;
    uint4* dst = reinterpret_cast<uint4*>(prm.o + row0 * D);
    for (int e = tid; e < chunks; e += 256) dst[e] = make_uint4(0, 0, 0, 0);
    if (prm.lse && tid < 64) prm.lse[row0 + tid] = -INFINITY;
    return;
  }
  const int T = (n + 1) >> 1;   // key tiles of two blocks

  if (warp == 2) {
    tmem_alloc(sbase + AttnSmem::kMisc, 256);
    tmem_relinquish();
  }
  if (D == 64) {   // V^T is padded to M = 128 rows of head dim with zeros
    for (int s = 0; s < kStages; ++s) {
      uint4* z = reinterpret_cast<uint4*>(sm + AttnSmem::kV + s * AttnSmem::kKStage + 16384);
      for (int e = tid; e < 16384 / 16; e += 256) z[e] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_misc[0];
  const uint32_t tS[2] = {tmem + 0u, tmem + 64u};
  const uint32_t tO = tmem + 128u;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(BAR_Q), 64 * D * 2);
      for (int h = 0; h < DH; ++h)
        tma_load_2d(sbase + AttnSmem::kQ + h * 8192, &tmQ, bar(BAR_Q), 64 * h, static_cast<int32_t>(row0));
      int armed[kStages];
      for (int s = 0; s < kStages; ++s) armed[s] = 0;
      for (int t = 0; t < T; ++t) {
        if (*s_abort) break;
        const int s = t % kStages;
        if (t >= kStages && !mbar_wait(bar(BAR_KVEMPTY + s), ((t / kStages) - 1) & 1)) {
          *s_abort = 1;
          break;
        }
        const int j0 = s_list[2 * t];
        const int j1 = (2 * t + 1 < n) ? s_list[2 * t + 1] : j0;   // odd tail: duplicate, masked in softmax
        const int32_t y0 = static_cast<int32_t>(bh * prm.N + static_cast<long long>(j0) * 64);
        const int32_t y1 = static_cast<int32_t>(bh * prm.N + static_cast<long long>(j1) * 64);
        const uint32_t kst = sbase + AttnSmem::kK + s * AttnSmem::kKStage;
        const uint32_t vst = sbase + AttnSmem::kV + s * AttnSmem::kKStage;
        mbar_expect_tx(bar(BAR_KFULL + s), 128 * D * 2);
        for (int h = 0; h < DH; ++h) {
          tma_load_2d(kst + h * 16384, &tmK, bar(BAR_KFULL + s), 64 * h, y0);
          tma_load_2d(kst + h * 16384 + 8192, &tmK, bar(BAR_KFULL + s), 64 * h, y1);
        }
        mbar_expect_tx(bar(BAR_VFULL + s), 128 * D * 2);
        for (int h = 0; h < DH; ++h) {
          tma_load_2d(vst + h * 16384, &tmV, bar(BAR_VFULL + s), 64 * h, y0);
          tma_load_2d(vst + h * 16384 + 8192, &tmV, bar(BAR_VFULL + s), 64 * h, y1);
        }
        armed[s] = t / kStages + 1;
      }
      // every load issued must land before the CTA can retire
      for (int s = 0; s < kStages; ++s) {
        if (armed[s] > 0) {
          mbar_wait(bar(BAR_KFULL + s), (armed[s] - 1) & 1);
          mbar_wait(bar(BAR_VFULL + s), (armed[s] - 1) & 1);
        }
      }
      mbar_wait(bar(BAR_Q), 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);   // A = K tile (K-major), B = Q (K-major)
      constexpr uint32_t idO = idesc_bf16(128, 64, 1, 1);   // A = V^T (MN-major), B = P^T (MN-major)
      const uint32_t qa = sbase + AttnSmem::kQ;
      bool ok = mbar_wait(bar(BAR_Q), 0);
      auto issue_pv = [&](int u) -> bool {
        const int s = u % kStages, b = u & 1;
        if (!mbar_wait(bar(BAR_PFULL + b), (u >> 1) & 1)) return false;
        if (!mbar_wait(bar(BAR_VFULL + s), (u / kStages) & 1)) return false;
        tc_fence_after();
        const uint32_t va = sbase + AttnSmem::kV + s * AttnSmem::kKStage;
        const uint32_t pa = sbase + AttnSmem::kP + b * AttnSmem::kPBuf;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = smem_desc(va + kk * 2048, 16384, 1024);
          const uint64_t bd = smem_desc(pa + kk * 2048, 16384, 1024);
          umma_f16(tO, ad, bd, idO, (u > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(BAR_PEMPTY + b));
        umma_commit(bar(BAR_KVEMPTY + s));
        return true;
      };
      int t = 0;
      for (; ok && t < T; ++t) {
        if (*s_abort) { ok = false; break; }
        const int s = t % kStages, b = t & 1;
        if (!mbar_wait(bar(BAR_KFULL + s), (t / kStages) & 1)) { ok = false; break; }
        if (t >= 2 && !mbar_wait(bar(BAR_SEMPTY + b), ((t >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka = sbase + AttnSmem::kK + s * AttnSmem::kKStage;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_f16(tS[b], smem_desc(ka + off, 16, 1024), smem_desc(qa + qoff, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(BAR_SFULL + b));
        if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(T - 1);
      if (ok) umma_commit(bar(BAR_OFULL));
      if (!ok) *s_abort = 1;
      // drain: all MMAs issued by this thread complete before teardown
      umma_commit(bar(BAR_DRAIN));
      mbar_wait(bar(BAR_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp - 4;                 // TMEM lane quarter
    const int t128 = tid - 128;
    const int r = 32 * q + lane;            // key row of S^T within the tile
    const uint32_t tl = static_cast<uint32_t>(32 * q) << 16;
    const float sc = prm.scale_log2;
    float* s_mref = s_final;                // [64] per-query reference max (CTA-uniform)
    float* s_alpha = s_final + 64;          // [64] rescale factors of the current tile
    float lpart[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) lpart[c] = 0.0f;
    bool bad = false;
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      if (!mbar_wait(bar(BAR_SFULL + b), (t >> 1) & 1)) bad = true;
      tc_fence_after();
      float x[64];
      {
        uint32_t u0[32], u1[32];
        tmem_ld32(tS[b] + tl, u0);
        tmem_ld32(tS[b] + tl + 32, u1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(u0[c]);
          x[c + 32] = __uint_as_float(u1[c]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(BAR_SEMPTY + b));
      const bool valid = (r < 64) || (2 * t + 1 < n);
#pragma unroll
      for (int c = 0; c < 64; ++c) x[c] = valid ? x[c] * sc : -INFINITY;

      bool rescale = (t == 0);
      if (t > 0) {
        float dmax = -INFINITY;
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 m4 = reinterpret_cast<const float4*>(s_mref)[c4];
          dmax = fmaxf(dmax, fmaxf(fmaxf(x[4 * c4] - m4.x, x[4 * c4 + 1] - m4.y),
                                   fmaxf(x[4 * c4 + 2] - m4.z, x[4 * c4 + 3] - m4.w)));
        }
        rescale = dmax > kRescaleLog2;
      }
      rescale = bar_red_or(rescale || bad);
      if (*s_abort) bad = true;
      if (rescale) {
        // per-query max over this tile's 128 keys -> new reference max and rescale factor
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float cm = warp_max_f32(x[c]);
          if (lane == (c & 31)) s_red[q * 64 + c] = cm;
        }
        named_bar_sync(1, 128);
        if (t128 < 64) {
          const int c = t128;
          const float tm = fmaxf(fmaxf(s_red[c], s_red[64 + c]), fmaxf(s_red[128 + c], s_red[192 + c]));
          if (t == 0) {
            s_mref[c] = tm;
            s_alpha[c] = 1.0f;
          } else {
            const float mo = s_mref[c];
            const float mn = fmaxf(mo, tm);
            s_alpha[c] = fast_exp2(mo - mn);
            s_mref[c] = mn;
          }
        }
        named_bar_sync(1, 128);
        if (t > 0) {
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 a4 = reinterpret_cast<const float4*>(s_alpha)[c4];
            lpart[4 * c4] *= a4.x;
            lpart[4 * c4 + 1] *= a4.y;
            lpart[4 * c4 + 2] *= a4.z;
            lpart[4 * c4 + 3] *= a4.w;
          }
          // O^T holds tiles 0..t-1 once PV(t-1) has completed
          if (!mbar_wait(bar(BAR_PEMPTY + ((t - 1) & 1)), ((t - 1) >> 1) & 1)) bad = true;
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t ov[32];
            tmem_ld32(tO + tl + 32 * h, ov);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * s_alpha[32 * h + c]);
            tmem_st32(tO + tl + 32 * h, ov);
          }
          tmem_wait_st();
          tc_fence_before();
        }
      }
      // P = 2^(x - mref), per-query partial sums, bf16 pack
      uint32_t pk[32];
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 m4 = reinterpret_cast<const float4*>(s_mref)[c4];
        const float p0 = fast_exp2(x[4 * c4] - m4.x);
        const float p1 = fast_exp2(x[4 * c4 + 1] - m4.y);
        const float p2 = fast_exp2(x[4 * c4 + 2] - m4.z);
        const float p3 = fast_exp2(x[4 * c4 + 3] - m4.w);
        lpart[4 * c4] += p0;
        lpart[4 * c4 + 1] += p1;
        lpart[4 * c4 + 2] += p2;
        lpart[4 * c4 + 3] += p3;
        pk[2 * c4] = pack_bf16x2(p0, p1);
        pk[2 * c4 + 1] = pack_bf16x2(p2, p3);
      }
      if (t >= 2 && !mbar_wait(bar(BAR_PEMPTY + b), ((t - 2) >> 1) & 1)) bad = true;
      // P^T row r (128 bytes) in the 128-byte-swizzled MN-major layout
      uint8_t* prow = sm + AttnSmem::kP + b * AttnSmem::kPBuf + r * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const int phys = c8 ^ (r & 7);
        *reinterpret_cast<uint4*>(prow + phys * 16) =
            make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
      }
      fence_async_smem();
      mbar_arrive(bar(BAR_PFULL + b));
      if (bad) *s_abort = 1;
      if (bar_red_or(bad)) break;
    }

    // ---- epilogue: per-query sums, O^T / l, bf16 store, log-sum-exp
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      float v = lpart[c];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == (c & 31)) s_lsum[q * 64 + c] = v;
    }
    named_bar_sync(1, 128);
    float* s_inv = s_red;                   // [64] 1 / l, reusing the max-exchange buffer
    if (t128 < 64) {
      const int c = t128;
      const float l = (s_lsum[c] + s_lsum[64 + c]) + (s_lsum[128 + c] + s_lsum[192 + c]);
      s_inv[c] = 1.0f / l;
      if (prm.lse) prm.lse[row0 + c] = (s_mref[c] + __log2f(l)) * 0.69314718055994530942f;
    }
    if (!mbar_wait(bar(BAR_OFULL), 0)) *s_abort = 1;
    tc_fence_after();
    named_bar_sync(1, 128);
    // O^T lanes = head-dim rows d = r; stage as [64 queries][D] bf16 in the (idle) K stage 0
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(sm + AttnSmem::kK);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t ov[32];
      tmem_ld32(tO + tl + 32 * h, ov);
      tmem_wait_ld();
      if (r < D) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          stage[(32 * h + c) * D + r] = __float2bfloat16_rn(__uint_as_float(ov[c]) * s_inv[32 * h + c]);
      }
    }
    tc_fence_before();
    named_bar_sync(1, 128);
    const uint4* src = reinterpret_cast<const uint4*>(stage);
    uint4* dst = reinterpret_cast<uint4*>(prm.o + row0 * D);
#pragma unroll
    for (int e = t128; e < 64 * D / 8; e += 128) dst[e] = src[e];
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace dbst
