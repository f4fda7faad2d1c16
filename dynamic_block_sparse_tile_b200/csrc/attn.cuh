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
// and keeps per-query partial sums; the per-query running max is a reference
// shared by the 128 key lanes, refreshed only when a tile exceeds it by more
// than kRescaleLog2 (exact: numerator and denominator share the reference).
//
// Warp roles (384 threads):
//   warp 0      TMA producer of Q and of the K ring (kKSlots tiles)
//   warp 1      MMA issuer (one thread): S(t+2) is issued as soon as the
//               softmax has read S(t), PV(t) as soon as P(t) is written
//   warp 2      TMEM allocation
//   warp 3      TMA producer of the V ring (kVSlots tiles)
//   warps 4..   kSoftWG softmax warpgroups; warpgroup g owns query columns
//               kCols*g .. kCols*g + kCols-1
// Warp 4+4g+q owns TMEM lanes 32q..32q+31.  The warpgroups own disjoint
// query columns of S^T, O^T and of the output, so each keeps its own running
// max, sums and rescaling decisions; several warpgroups per SM sub-partition
// hide the latency of TMEM loads, exponentials and the per-tile vote.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace dbst {

constexpr int kKSlots = 3;
constexpr int kVSlots = 2;
constexpr int kSoftWG = 4;                       // softmax warpgroups
constexpr int kCols = 64 / kSoftWG;              // query columns per softmax warpgroup
constexpr int kAttnThreads = 128 + 128 * kSoftWG;
constexpr float kRescaleLog2 = 16.0f;
constexpr int kSBufs = 4;                        // S^T buffers in TMEM (tile t uses buffer t % 4)

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
  static constexpr int kTile = 32768;                   // one K or V tile: 2 D-halves x [128 keys x 128 B]
  static constexpr int kK = kQ + 16384;                 // K ring
  static constexpr int kV = kK + kKSlots * kTile;       // V ring (D=64: half 1 = zeros)
  static constexpr int kP = kV + kVSlots * kTile;       // P^T buffers: [128 keys x 64 queries] bf16
  static constexpr int kPBuf = 16384;
  static constexpr int kList = kP + 2 * kPBuf;          // compacted key-block list, int16 x 4096
  static constexpr int kRed = kList + 8192;             // float [wg][4 warps][kCols] column max exchange
  static constexpr int kLsum = kRed + 1024;             // float [wg][4][kCols] column sums
  static constexpr int kFinal = kLsum + 1024;           // float [64] 1/l, float [wg][kCols] rescale factors
  static constexpr int kBars = kFinal + 512;            // mbarriers
  static constexpr int kMisc = kBars + 256;             // tmem base, list length, abort flags
  static constexpr int kBytes = kMisc + 64;
};

// barrier slots (8 bytes each)
enum {
  BAR_Q = 0,
  BAR_KFULL = 1,
  BAR_KEMPTY = BAR_KFULL + kKSlots,
  BAR_VFULL = BAR_KEMPTY + kKSlots,
  BAR_VEMPTY = BAR_VFULL + kVSlots,
  BAR_SFULL = BAR_VEMPTY + kVSlots,   // + kSBufs
  BAR_SEMPTY = BAR_SFULL + kSBufs,    // one arrival per softmax thread
  BAR_PFULL = BAR_SEMPTY + kSBufs,    // one arrival per softmax thread
  BAR_PEMPTY = BAR_PFULL + 2,
  BAR_OFULL = BAR_PEMPTY + 2,
  BAR_DRAIN = BAR_OFULL + 1,
  BAR_COUNT = BAR_DRAIN + 1
};
static_assert(BAR_COUNT * 8 <= 256, "barrier area");

// OR-reduction of a predicate over one softmax warpgroup (named barrier 1 + wg, 128 threads).
__device__ __forceinline__ bool wg_vote_or(int wg, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(1 + wg)
      : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int DH = D / 64;                 // 128-byte column halves per token row
  constexpr int NWARPS = kAttnThreads / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  int16_t* s_list = reinterpret_cast<int16_t*>(sm + AttnSmem::kList);
  float* s_red = reinterpret_cast<float*>(sm + AttnSmem::kRed);
  float* s_lsum = reinterpret_cast<float*>(sm + AttnSmem::kLsum);
  float* s_inv = reinterpret_cast<float*>(sm + AttnSmem::kFinal);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(sm + AttnSmem::kMisc);
  volatile uint32_t* s_abort = s_misc + 2;   // set by the producers / MMA issuer
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
      if ((b >= BAR_SEMPTY && b < BAR_SEMPTY + kSBufs) || b == BAR_PFULL || b == BAR_PFULL + 1) cnt = 128 * kSoftWG;
      mbar_init(bar(b), cnt);
    }
    fence_mbar_init();
    for (int i = 1; i < 8; ++i) s_misc[i] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n_raw; base += kAttnThreads) {
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
      for (int w = 0; w < NWARPS; ++w) tot += __float_as_int(s_red[w]);
      s_misc[1] += tot;
    }
    __syncthreads();
  }
  const int n = static_cast<int>(s_misc[1]);

  if (n == 0) {   // no kept key block: o = 0, lse = -inf
    const int chunks = 64 * D / 8;
    uint4* dst = reinterpret_cast<uint4*>(prm.o + row0 * D);
    for (int e = tid; e < chunks; e += kAttnThreads) dst[e] = make_uint4(0, 0, 0, 0);
    if (prm.lse && tid < 64) prm.lse[row0 + tid] = -INFINITY;
    return;
  }
  const int T = (n + 1) >> 1;   // key tiles of two blocks

  if (warp == 2) {
    tmem_alloc(sbase + AttnSmem::kMisc, 512);
    tmem_relinquish();
  }
  if (D == 64) {   // V^T is padded to M = 128 rows of head dim with zeros
    for (int s = 0; s < kVSlots; ++s) {
      uint4* z = reinterpret_cast<uint4*>(sm + AttnSmem::kV + s * AttnSmem::kTile + 16384);
      for (int e = tid; e < 16384 / 16; e += kAttnThreads) z[e] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_misc[0];
  const uint32_t tS0 = tmem;              // S^T buffer k at TMEM columns 64k
  const uint32_t tO = tmem + 256u;

  auto tile_rows = [&](int t, int32_t& y0, int32_t& y1) {
    const int j0 = s_list[2 * t];
    const int j1 = (2 * t + 1 < n) ? s_list[2 * t + 1] : j0;   // odd tail: duplicate, masked in softmax
    y0 = static_cast<int32_t>(bh * prm.N + static_cast<long long>(j0) * 64);
    y1 = static_cast<int32_t>(bh * prm.N + static_cast<long long>(j1) * 64);
  };

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ TMA producers (K ring / V ring)
    if (lane == 0) {
      const bool isK = (warp == 0);
      const CUtensorMap* map = isK ? &tmK : &tmV;
      const int slots = isK ? kKSlots : kVSlots;
      const int full0 = isK ? BAR_KFULL : BAR_VFULL;
      const int empty0 = isK ? BAR_KEMPTY : BAR_VEMPTY;
      const uint32_t ring = sbase + (isK ? AttnSmem::kK : AttnSmem::kV);
      tma_prefetch_desc(map);
      if (isK) {
        tma_prefetch_desc(&tmQ);
        mbar_expect_tx(bar(BAR_Q), 64 * D * 2);
        for (int h = 0; h < DH; ++h)
          tma_load_2d(sbase + AttnSmem::kQ + h * 8192, &tmQ, bar(BAR_Q), 64 * h, static_cast<int32_t>(row0));
      }
      int armed[kKSlots] = {0, 0, 0};
      for (int t = 0; t < T; ++t) {
        if (*s_abort) break;
        const int s = t % slots;
        if (t >= slots && !mbar_wait(bar(empty0 + s), ((t / slots) - 1) & 1)) {
          *s_abort = 1;
          break;
        }
        int32_t y0, y1;
        tile_rows(t, y0, y1);
        const uint32_t dst = ring + s * AttnSmem::kTile;
        mbar_expect_tx(bar(full0 + s), 128 * D * 2);
        for (int h = 0; h < DH; ++h) {
          tma_load_2d(dst + h * 16384, map, bar(full0 + s), 64 * h, y0);
          tma_load_2d(dst + h * 16384 + 8192, map, bar(full0 + s), 64 * h, y1);
        }
        armed[s] = t / slots + 1;
      }
      // every load issued must land before the CTA can retire
      for (int s = 0; s < slots; ++s)
        if (armed[s] > 0) mbar_wait(bar(full0 + s), (armed[s] - 1) & 1);
      if (isK) mbar_wait(bar(BAR_Q), 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (operands stay warp-uniform); one elected
    // lane issues each tcgen05.mma / commit.  Wait results are agreed on with
    // __all_sync so that control flow never diverges inside the warp.
    constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);   // A = K tile (K-major), B = Q (K-major)
    constexpr uint32_t idO = idesc_bf16(128, 64, 1, 1);   // A = V^T (MN-major), B = P^T (MN-major)
    const uint64_t dQ = smem_desc(sbase + AttnSmem::kQ, 16, 1024);
    const uint64_t dK = smem_desc(sbase + AttnSmem::kK, 16, 1024);
    const uint64_t dV = smem_desc(sbase + AttnSmem::kV, 16384, 1024);
    const uint64_t dP = smem_desc(sbase + AttnSmem::kP, 16384, 1024);
    auto wait_all = [&](int slot, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar(slot), parity));
    };
    auto issue_s = [&](int t) -> bool {
      const int s = t % kKSlots, b = t % kSBufs;
      if (!wait_all(BAR_KFULL + s, (t / kKSlots) & 1)) return false;
      if (t >= kSBufs && !wait_all(BAR_SEMPTY + b, ((t / kSBufs) - 1) & 1)) return false;
      tc_fence_after();
      const uint64_t ka = dK + static_cast<uint64_t>((s * AttnSmem::kTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        const uint32_t qoff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
        umma_f16_elect(tS0 + 64u * b, ka + off, dQ + qoff, idS, kk > 0 ? 1u : 0u);
      }
      umma_commit_elect(bar(BAR_SFULL + b));
      umma_commit_elect(bar(BAR_KEMPTY + s));
      return true;
    };
    auto issue_pv = [&](int u) -> bool {
      const int sv = u % kVSlots, b = u & 1;
      if (!wait_all(BAR_PFULL + b, (u >> 1) & 1)) return false;
      if (!wait_all(BAR_VFULL + sv, (u / kVSlots) & 1)) return false;
      tc_fence_after();
      const uint64_t va = dV + static_cast<uint64_t>((sv * AttnSmem::kTile) >> 4);
      const uint64_t pa = dP + static_cast<uint64_t>((b * AttnSmem::kPBuf) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) umma_f16_elect(tO, va + kk * 128, pa + kk * 128, idO, (u > 0 || kk > 0) ? 1u : 0u);
      umma_commit_elect(bar(BAR_PEMPTY + b));
      umma_commit_elect(bar(BAR_VEMPTY + sv));
      return true;
    };
    bool ok = wait_all(BAR_Q, 0);
    if (ok) ok = issue_s(0);
    if (ok && T > 1) ok = issue_s(1);
    for (int u = 0; ok && u < T; ++u) {
      if (__any_sync(0xffffffffu, *s_abort != 0)) { ok = false; break; }
      if (u + 2 < T && !issue_s(u + 2)) { ok = false; break; }
      if (!issue_pv(u)) { ok = false; break; }
    }
    if (ok) umma_commit_elect(bar(BAR_OFULL));
    if (!ok && lane == 0) *s_abort = 1;
    // drain: all MMAs issued by this warp complete before teardown
    umma_commit_elect(bar(BAR_DRAIN));
    mbar_wait(bar(BAR_DRAIN), 0);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 4) >> 2;           // warpgroup: query columns c0 .. c0 + kCols - 1
    const int q = warp & 3;                   // TMEM lane quarter
    const int twg = tid - 128 - 128 * wg;     // thread index within the warpgroup
    const int r = 32 * q + lane;              // key row of S^T within the tile (= head-dim row of O^T)
    const int c0 = kCols * wg;
    const uint32_t tl = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t barid = 1 + wg;
    const float sc = prm.scale_log2;
    volatile uint32_t* wg_abort = s_misc + 3 + wg;
    float* red = s_red + wg * 4 * kCols;      // [4 warps][kCols]
    float* lsum = s_lsum + wg * 4 * kCols;
    float* alpha_s = s_inv + 64 + kCols * wg; // [kCols] rescale factors of this warpgroup
    float mref[kCols], lpart[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      lpart[c] = 0.0f;
      mref[c] = 0.0f;
    }
    uint8_t* const prow_base = sm + AttnSmem::kP + r * 128;
    // P = 2^min(d, kRescaleLog2): per-query sums and this warpgroup's chunk of P^T row r (128-byte
    // swizzle).  The clamp only bites on tiles that trigger a rescale; their contributions are then
    // subtracted again, each at most 2^kRescaleLog2 and added to a sum that is rescaled by at least
    // that factor, so the sum keeps its relative accuracy.
    auto emit_p = [&](int b, const float (&d)[kCols], float sign) {
      uint32_t pk[kCols / 2];
#pragma unroll
      for (int c = 0; c < kCols / 2; ++c) {
        const float p0 = fast_exp2(fminf(d[2 * c], kRescaleLog2));
        const float p1 = fast_exp2(fminf(d[2 * c + 1], kRescaleLog2));
        lpart[2 * c] = fmaf(sign, p0, lpart[2 * c]);
        lpart[2 * c + 1] = fmaf(sign, p1, lpart[2 * c + 1]);
        pk[c] = pack_bf16x2(p0, p1);
      }
      if (sign > 0.0f) {
        uint8_t* prow = prow_base + b * AttnSmem::kPBuf;
#pragma unroll
        for (int cc = 0; cc < kCols / 8; ++cc) {
          const int phys = (kCols / 8 * wg + cc) ^ (r & 7);
          *reinterpret_cast<uint4*>(prow + phys * 16) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
      }
    };
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      const int sb = t % kSBufs;
      bool bad = !mbar_wait(bar(BAR_SFULL + sb), (t / kSBufs) & 1);
      // P^T buffer b is free once PV(t-2) has read it
      if (t >= 2 && !mbar_wait(bar(BAR_PEMPTY + b), ((t - 2) >> 1) & 1)) bad = true;
      tc_fence_after();
      // d = scaled logit - reference max (log2 units); rows of an absent second block are -inf
      float d[kCols];
      {
        uint32_t u[kCols];
        tmem_ld16(tS0 + 64u * sb + tl + c0, u);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kCols; ++c) d[c] = fmaf(__uint_as_float(u[c]), sc, -mref[c]);
      }
      if (q >= 2 && 2 * t + 1 >= n) {
#pragma unroll
        for (int c = 0; c < kCols; ++c) d[c] = -INFINITY;
      }
      // speculative pass with the current reference; the tile max decides whether it stands
      float dmax = -INFINITY;
      if (t > 0) {
#pragma unroll
        for (int c = 0; c < kCols; ++c) dmax = fmaxf(dmax, d[c]);
        emit_p(b, d, 1.0f);
      }
      if (bad) *wg_abort = 1;
      const bool need = wg_vote_or(wg, t == 0 || dmax > kRescaleLog2 || bad);
      if (*wg_abort) break;   // written before the vote by this warpgroup only: uniform
      if (need) {
        if (t > 0) emit_p(b, d, -1.0f);   // undo the speculative sums
        // per-query max over this tile's 128 keys -> new reference, rescale factors
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
          const float cm = warp_max_f32(d[c]);
          if (lane == c) red[q * kCols + c] = cm;
        }
        named_bar_sync(barid, 128);
#pragma unroll
        for (int c4 = 0; c4 < kCols / 4; ++c4) {
          float4 m4 = reinterpret_cast<const float4*>(red)[c4];
#pragma unroll
          for (int qq = 1; qq < 4; ++qq) {
            const float4 o4 = reinterpret_cast<const float4*>(red + qq * kCols)[c4];
            m4.x = fmaxf(m4.x, o4.x); m4.y = fmaxf(m4.y, o4.y);
            m4.z = fmaxf(m4.z, o4.z); m4.w = fmaxf(m4.w, o4.w);
          }
          const float tm[4] = {m4.x, m4.y, m4.z, m4.w};   // tile max relative to the old reference
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * c4 + e;
            const float shift = (t == 0) ? tm[e] : fmaxf(tm[e], 0.0f);
            mref[c] += shift;
            d[c] -= shift;
            if (t > 0) {
              const float a = fast_exp2(-shift);
              lpart[c] *= a;
              if (q == 0 && lane == c) alpha_s[c] = a;
            }
          }
        }
        if (t > 0) {
          // O^T holds tiles 0..t-1 once PV(t-1) has completed
          if (!mbar_wait(bar(BAR_PEMPTY + ((t - 1) & 1)), ((t - 1) >> 1) & 1)) *wg_abort = 1;
          named_bar_sync(barid, 128);   // alpha_s visible
          tc_fence_after();
          uint32_t ov[kCols];
          tmem_ld16(tO + tl + c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < kCols / 4; ++c4) {
            const float4 a4 = reinterpret_cast<const float4*>(alpha_s)[c4];
            ov[4 * c4] = __float_as_uint(__uint_as_float(ov[4 * c4]) * a4.x);
            ov[4 * c4 + 1] = __float_as_uint(__uint_as_float(ov[4 * c4 + 1]) * a4.y);
            ov[4 * c4 + 2] = __float_as_uint(__uint_as_float(ov[4 * c4 + 2]) * a4.z);
            ov[4 * c4 + 3] = __float_as_uint(__uint_as_float(ov[4 * c4 + 3]) * a4.w);
          }
          tmem_st16(tO + tl + c0, ov);
          tmem_wait_st();
        }
        emit_p(b, d, 1.0f);
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(bar(BAR_SEMPTY + sb));
      mbar_arrive(bar(BAR_PFULL + b));
    }

    // ---- epilogue: per-query sums, O^T / l, bf16 store, log-sum-exp
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      float v = lpart[c];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == c) lsum[q * kCols + c] = v;
    }
    named_bar_sync(barid, 128);
    if (twg < kCols) {
      const int c = twg;
      const float l = (lsum[c] + lsum[kCols + c]) + (lsum[2 * kCols + c] + lsum[3 * kCols + c]);
      s_inv[c0 + c] = 1.0f / l;
      float m = 0.0f;
#pragma unroll
      for (int cc = 0; cc < kCols; ++cc)
        if (cc == c) m = mref[cc];
      if (prm.lse) prm.lse[row0 + c0 + c] = (m + __log2f(l)) * 0.69314718055994530942f;
    }
    if (!mbar_wait(bar(BAR_OFULL), 0)) *s_abort = 1;
    tc_fence_after();
    named_bar_sync(barid, 128);
    // O^T lanes = head-dim rows d = r; stage this warpgroup's queries as [query][D] bf16 in K slot 0
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(sm + AttnSmem::kK);
    {
      uint32_t ov[kCols];
      tmem_ld16(tO + tl + c0, ov);
      tmem_wait_ld();
      if (r < D) {
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          stage[(c0 + c) * D + r] = __float2bfloat16_rn(__uint_as_float(ov[c]) * s_inv[c0 + c]);
      }
    }
    tc_fence_before();
    named_bar_sync(barid, 128);
    const uint4* src = reinterpret_cast<const uint4*>(stage + c0 * D);
    uint4* dst = reinterpret_cast<uint4*>(prm.o + (row0 + c0) * D);
#pragma unroll
    for (int e = twg; e < kCols * D / 8; e += 128) dst[e] = src[e];
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dbst
