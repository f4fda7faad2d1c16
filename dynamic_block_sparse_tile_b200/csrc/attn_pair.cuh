// Block-sparse exact softmax attention on sm_100a tensor cores ("Expansion"
// step on the NABLA page: attention over the tokens of the kept 64 x 64 tile
// pairs only).
//
// Formulation ("query pairs").  One CTA owns two 64-token query blocks qa, qb
// (the pair the caller's pair list names, else neighbours one tile step apart)
// as one 128-row query tile, and walks the union of their kept key blocks two
// at a time:
//     S[128 queries x 128 keys] = Q[128 x D] . K_tile[128 x D]^T      (tcgen05 SS, M=128, N=128)
//     O[128 queries x D]       += P[128 x 128 keys] . V_tile[128 x D]  (tcgen05 TS: P read from TMEM)
// A key block kept by only one of the two query blocks is masked (P = 0) in
// the other block's 64 rows.  With a logit offset per (query block, key block) (SIP's log(1/pi) on
// the AB-Attention page, section "Les trois techniques"), x = s * scale + offset enters the row max
// and the exponent in place of s * scale: the exponential warps fold it into the constant of their
// fused multiply-add, so offsets cost two loads per warp per tile, fetched a tile ahead.
//
// TMEM (512 columns): O at 0..D-1, S buffers at 128 and 256, P buffers (bf16
// pairs, 64 columns each) at 384 and 448.  Because P has its own buffers, S(t+2)
// is issued as soon as the softmax warps have read S(t) into registers, so the
// tensor core computes the next logits while the exponentials of this tile run.
//
// Warp roles (480 threads; a warp that reads TMEM sees lanes 32*(w%4) .. +31 only):
//   warps 0-3   row-max warps: warp q reads all 128 columns of S(t) for query rows 32q .. +31,
//               sets each row's reference max for tile t (moving it, and rescaling the rows of O,
//               when the tile's max runs more than kPairRescale above it) and publishes it.  They
//               run about a tile ahead of the exponential warps.
//   warps 4-11  exponential warps: warp w covers rows 32*(w%4) .. +31 and key block hc = (w-4)/4
//               of each tile (S columns 64*hc .. +63); P = 2^(x*scale - m) as bf16 pairs into the
//               P buffer, and a partial row sum.
//   warp 12     TMEM owner and MMA issuer (whole warp, one elected lane issues)
//   warp 13     TMA producer of Q and the K ring (lane 0)
//   warp 14     TMA producer of the V ring (lane 0); a warp of its own, so that its waits for
//               free V slots never hold up the K loads
//
// Waits between roles are bounded by a run-time limit (PairParams::wait_limit, default about one
// second); one that runs out records DBST_ETIMEOUT and the CTA abandons its work: producers stop
// issuing, the softmax roles run out their loops without waiting, and each role waits (with the
// default limit) for the copies and products it issued itself before the CTA frees TMEM and exits.
//
// CTAs run in grid order: head by head, each head's pairs in the order of the pair list (the
// pairing lists them longest first, so the short pairs fill the end of the launch).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "reorder.cuh"

namespace dbst {

constexpr int kPairThreads = 480;
constexpr int kPairKSlots = 3;
constexpr int kPairVSlots = 2;
// A tile whose row max exceeds the running reference by more than this (log2
// units) moves the reference and rescales the row; below it the stale reference
// is kept (exact: the numerator and the denominator share it).  P <= 2^kPairRescale.
constexpr float kPairRescale = 16.0f;

struct PairParams {
  const int32_t* kv_count;   // [BH*NB]; null => dense (every list is 0..NB-1)
  const int16_t* kv_idx;     // [BH*NB*NB]
  const float* offsets;      // [BH][NB][NB] logit offset (natural log) per (query block, key block), read at
                             // kept blocks only; null => none
  __nv_bfloat16* o;          // [BH, N, D], tile or raster order (RASTER)
  float* lse;                // [BH, N] in the same order, or null
  int NB, N;
  const int32_t* pairs;      // [BH][pairs_per_head] qa | qb << 16 (qb 0xFFFF: none), or null
  int pair_stride;           // without a pair list: qb = qa + pair_stride
  int pairs_per_head;
  float scale_log2;          // softmax scale * log2(e)
  long long wait_limit;      // cycles a wait between roles may take before the CTA gives up (0: default)
  TileGeo tg;                // token grid and tile shape (raster layout only)
};

struct PairSmem {
  static constexpr int kQ = 0;                            // Q: D-halves x [128 rows x 128 B]
  static constexpr int kTile = 32768;                     // K or V tile: D-halves x [128 keys x 128 B]
  static constexpr int kK = kQ + 32768;
  static constexpr int kV = kK + kPairKSlots * kTile;
  static constexpr int kUnion = kV + kPairVSlots * kTile; // int32 x 4096: j | inA<<16 | inB<<17
  static constexpr int kWords = kUnion + 16384;           // u32 [2][128] bitmasks of the two lists
  static constexpr int kScan = kWords + 1024;             // int [128] word offsets
  static constexpr int kRing = kScan + 512;               // float2 [2 tile parities][128 rows]: (m, a)
  static constexpr int kLsum = kRing + 2048;              // float [2 sums][2 halves][128 rows]
  static constexpr int kBars = kLsum + 2048;
  static constexpr int kMisc = kBars + 256;
  static constexpr int kBytes = kMisc + 64;
};

enum {
  PB_Q = 0,
  PB_KFULL = 1,
  PB_KEMPTY = PB_KFULL + kPairKSlots,
  PB_VFULL = PB_KEMPTY + kPairKSlots,
  PB_VEMPTY = PB_VFULL + kPairVSlots,
  PB_SFULL = PB_VEMPTY + kPairVSlots,   // [2] S(t) in buffer t&1 is complete
  PB_SEMPTY = PB_SFULL + 2,             // [2] 384 arrivals: S(t) has been read
  PB_PFULL = PB_SEMPTY + 2,             // [2] 384 arrivals: P(t) is in buffer t&1, O rescaled for it
  PB_PVDONE = PB_PFULL + 2,             // [2] PV(t) has completed (P buffer t&1 free, O current)
  PB_MREADY = PB_PVDONE + 2,            // [2][4] 32 arrivals: row references of tile t, lane quarter q
  PB_DRAIN = PB_MREADY + 8,
  PB_COUNT = PB_DRAIN + 1
};
static_assert(PB_COUNT * 8 <= 256, "barrier area");

constexpr uint32_t kTmemO = 0, kTmemS = 128, kTmemP = 384;

__device__ __forceinline__ void umma_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// RASTER = false: q, k, v, o are in tile order (block j = rows 64j .. 64j+63 of a head), loaded
// with 2-D boxes.  RASTER = true: they are in the caller's raster order; the tile reorder is done
// by the loads themselves (5-D boxes tx x ty x tt tokens x 64 channels land in shared memory in
// exactly the tile-ordered layout) and by the epilogue, which writes o and lse rows in raster
// order.  Both produce bit-identical results.
// OFFSETS: the kernel reads PairParams::offsets (compiled apart so that the common case carries no
// offset bookkeeping).
template <int D, bool RASTER, bool OFFSETS = false>
__global__ void __launch_bounds__(kPairThreads, 1)
    pair_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const PairParams prm) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int DH = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  int32_t* s_union = reinterpret_cast<int32_t*>(sm + PairSmem::kUnion);
  uint32_t* s_words = reinterpret_cast<uint32_t*>(sm + PairSmem::kWords);
  int32_t* s_scan = reinterpret_cast<int32_t*>(sm + PairSmem::kScan);
  float2* s_ring = reinterpret_cast<float2*>(sm + PairSmem::kRing);
  float* s_lsum = reinterpret_cast<float*>(sm + PairSmem::kLsum);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(sm + PairSmem::kMisc);
  volatile uint32_t* s_abort = s_misc + 2;
  auto bar = [&](int slot) -> uint32_t { return sbase + PairSmem::kBars + 8u * slot; };
  // limit of a wait between roles; read only on a wait's slow path, so it holds no register in the loops
  auto limit = [&]() -> long long { return prm.wait_limit > 0 ? prm.wait_limit : kWaitLimitCycles; };
  // Bounded wait used inside the softmax loops.  The abort flag is read only when the phase is
  // not already complete, so a wait that succeeds at once costs one barrier test; `live` turns
  // false for good once this warp times out or sees another role's abort, and later waits are
  // then skipped so the warp runs its remaining iterations without blocking.
  auto wait_live = [&](uint32_t mb, uint32_t parity, bool& live) {
    if (!live || mbar_try(mb, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try(mb, parity)) {
      if (*s_abort) { live = false; return; }
      if (clock64() - t0 > limit()) {
        record_error(kErrTimeout);
        *s_abort = 1;
        live = false;
        return;
      }
    }
  };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NB = prm.NB, NW = (NB + 31) >> 5;
  const long long bh = blockIdx.x / prm.pairs_per_head;
  const int pi = blockIdx.x - static_cast<int>(bh * prm.pairs_per_head);
  int qa, qb;
  if (prm.pairs != nullptr) {
    const int32_t ent = prm.pairs[bh * prm.pairs_per_head + pi];
    qa = ent & 0xFFFF;
    qb = (ent >> 16) & 0xFFFF;
    if (qa >= NB || (qb >= NB && qb != 0xFFFF)) {   // not a block of this head: report, compute nothing
      if (threadIdx.x == 0) record_error(kErrBounds);
      return;
    }
  } else {
    const int ps = prm.pair_stride;
    qa = (pi / ps) * 2 * ps + (pi % ps);
    qb = qa + ps;
  }
  const bool has_b = qb < NB;
  // global row of row rr (0..63) of query block blk of this head
  auto out_row = [&](int blk, int rr) -> long long {
    if constexpr (RASTER) return bh * prm.N + tiled_to_raster(blk * 64 + rr, prm.tg);
    else return bh * prm.N + static_cast<long long>(blk) * 64 + rr;
  };
  // TMA load of block blk's channels 64h .. 64h+63 (8 KB) into shared memory
  auto load_block = [&](uint32_t dst, const CUtensorMap* map, uint32_t mbar, int blk, int h) {
    if constexpr (RASTER) {
      const int Tx = blk % prm.tg.nX, Ty = (blk / prm.tg.nX) % prm.tg.nY, Tt = blk / (prm.tg.nX * prm.tg.nY);
      tma_load_5d(dst, map, mbar, 64 * h, Tx * prm.tg.tx, Ty * prm.tg.ty, Tt * prm.tg.tt, static_cast<int32_t>(bh));
    } else {
      tma_load_2d(dst, map, mbar, 64 * h, static_cast<int32_t>(bh * prm.N + static_cast<long long>(blk) * 64));
    }
  };

  // ---- union of the two lists as bitmasks -> ascending entries with membership flags
  for (int w = tid; w < 2 * 128; w += kPairThreads) s_words[w] = 0u;
  if (tid == 0) {
    for (int b = 0; b < PB_COUNT; ++b) {
      uint32_t n = 1u;
      if (b >= PB_SEMPTY && b < PB_PVDONE) n = 384u;
      if (b >= PB_MREADY && b < PB_DRAIN) n = 32u;
      mbar_init(bar(b), n);
    }
    fence_mbar_init();
    for (int i = 1; i < 16; ++i) s_misc[i] = 0;
  }
  __syncthreads();
  // Work that does not depend on the lists starts at once: the Q tiles' loads and the TMEM
  // allocation overlap the list reads below.
  if (warp == 13 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    mbar_expect_tx(bar(PB_Q), 128 * D * 2);
    for (int h = 0; h < DH; ++h) {
      load_block(sbase + PairSmem::kQ + h * 16384, &tmQ, bar(PB_Q), qa, h);
      load_block(sbase + PairSmem::kQ + h * 16384 + 8192, &tmQ, bar(PB_Q), has_b ? qb : qa, h);
    }
  }
  if (warp == 12) {
    tmem_alloc(sbase + PairSmem::kMisc, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  // Both lists: both counts first, then all entries in one pass (two independent chains of loads).
  int n0 = NB, n1 = has_b ? NB : 0;
  const int16_t* g0 = nullptr;
  const int16_t* g1 = nullptr;
  if (prm.kv_count != nullptr) {
    n0 = prm.kv_count[bh * NB + qa];
    n1 = has_b ? prm.kv_count[bh * NB + qb] : 0;
    g0 = prm.kv_idx + (bh * NB + qa) * static_cast<long long>(NB);
    g1 = prm.kv_idx + (bh * NB + (has_b ? qb : qa)) * static_cast<long long>(NB);
    if (n0 < 0 || n0 > NB || n1 < 0 || n1 > NB) {
      if (tid == 0) record_error(kErrBounds);
      n0 = min(max(n0, 0), NB);
      n1 = min(max(n1, 0), NB);
    }
  }
  for (int e = tid; e < n0 + n1; e += kPairThreads) {
    const int side = e >= n0;
    const int ei = side ? e - n0 : e;
    const int16_t* gl = side ? g1 : g0;
    const int j = gl ? static_cast<int>(gl[ei]) : ei;
    if (j < 0 || j >= NB) {
      record_error(kErrBounds);
      continue;
    }
    atomicOr(&s_words[side * 128 + (j >> 5)], 1u << (j & 31));
  }
  __syncthreads();
  if (warp == 0) {   // exclusive scan of the union's popcounts over NW <= 128 words
    int cnt[4], tot = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int w = 4 * lane + e;
      cnt[e] = (w < NW) ? __popc(s_words[w] | s_words[128 + w]) : 0;
      tot += cnt[e];
    }
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - tot;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s_scan[4 * lane + e] = run;
      run += cnt[e];
    }
    if (lane == 31) s_misc[1] = static_cast<uint32_t>(incl);
  }
  __syncthreads();
  for (int w = tid; w < NW; w += kPairThreads) {
    const uint32_t wa = s_words[w], wb = s_words[128 + w];
    uint32_t u = wa | wb;
    int pos = s_scan[w];
    while (u) {
      const int b = __ffs(u) - 1;
      u &= u - 1u;
      s_union[pos++] = (32 * w + b) | (static_cast<int>((wa >> b) & 1u) << 16) | (static_cast<int>((wb >> b) & 1u) << 17);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_misc[0];
  const int nu = static_cast<int>(s_misc[1]);
  if (nu == 0) {   // neither block keeps anything: o = 0, lse = -inf
    // the Q loads are in flight and TMEM is held: let the one land and free the other
    if (warp == 13 && lane == 0) mbar_wait(bar(PB_Q), 0);
    if (warp == 12) tmem_dealloc(tmem, 512);
    for (int e = tid; e < 64 * D / 8; e += kPairThreads) {
      const int rr = e / (D / 8), c = e % (D / 8);
      reinterpret_cast<uint4*>(prm.o + out_row(qa, rr) * D)[c] = make_uint4(0, 0, 0, 0);
      if (has_b) reinterpret_cast<uint4*>(prm.o + out_row(qb, rr) * D)[c] = make_uint4(0, 0, 0, 0);
    }
    if (prm.lse && tid < 64) {
      prm.lse[out_row(qa, tid)] = -INFINITY;
      if (has_b) prm.lse[out_row(qb, tid)] = -INFINITY;
    }
    return;
  }
  const int T = (nu + 1) >> 1;
  // Logit offsets: the row of offsets of query block qa (side 0) or qb (side 1), null without offsets
  // (or for the absent second block); offset_of(row, e) is union entry e's offset in log2 units, 0 past
  // the union's end or without offsets.
  auto offset_row = [&](int side) -> const float* {
    if (!OFFSETS || prm.offsets == nullptr || (side == 1 && !has_b)) return nullptr;
    return prm.offsets + (bh * NB + (side ? qb : qa)) * static_cast<long long>(NB);
  };
  auto offset_of = [&](const float* orow, int e) -> float {
    if constexpr (!OFFSETS) return 0.0f;
    return (orow != nullptr && e < nu) ? __ldg(orow + (s_union[e] & 0xFFFF)) * 1.4426950408889634f : 0.0f;
  };

  if (warp == 13 || warp == 14) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool isK = (warp == 13);
      const CUtensorMap* map = isK ? &tmK : &tmV;
      const int slots = isK ? kPairKSlots : kPairVSlots;
      const int full0 = isK ? PB_KFULL : PB_VFULL;
      const int empty0 = isK ? PB_KEMPTY : PB_VEMPTY;
      const uint32_t ring = sbase + (isK ? PairSmem::kK : PairSmem::kV);
      tma_prefetch_desc(map);
      int armed[kPairKSlots] = {0, 0, 0};
      for (int t = 0; t < T; ++t) {
        if (*s_abort) break;
        const int s = t % slots;
        if (t >= slots && !mbar_wait_lim(bar(empty0 + s), ((t / slots) - 1) & 1, limit())) {
          *s_abort = 1;
          break;
        }
        const int j0 = s_union[2 * t] & 0xFFFF;
        const int j1 = (2 * t + 1 < nu) ? (s_union[2 * t + 1] & 0xFFFF) : j0;   // odd tail: duplicate, masked
        const uint32_t dst = ring + s * PairSmem::kTile;
        mbar_expect_tx(bar(full0 + s), 128 * D * 2);
        for (int h = 0; h < DH; ++h) {
          load_block(dst + h * 16384, map, bar(full0 + s), j0, h);
          load_block(dst + h * 16384 + 8192, map, bar(full0 + s), j1, h);
        }
        armed[s] = t / slots + 1;
      }
      for (int s = 0; s < slots; ++s)
        if (armed[s] > 0) mbar_wait(bar(full0 + s), (armed[s] - 1) & 1);
      if (isK) mbar_wait(bar(PB_Q), 0);
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);   // A = Q (K-major), B = K tile (K-major)
    constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);     // A = P in TMEM, B = V tile (MN-major)
    const uint64_t dQ = smem_desc(sbase + PairSmem::kQ, 16, 1024);
    const uint64_t dK = smem_desc(sbase + PairSmem::kK, 16, 1024);
    const uint64_t dV = smem_desc(sbase + PairSmem::kV, 16384, 1024);
    auto wait_all = [&](int slot, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_lim(bar(slot), parity, limit()));
    };
    // S(t) -> S buffer t&1, once the softmax has read S(t-2) out of it.
    auto issue_s = [&](int t) -> bool {
      const int s = t % kPairKSlots, b = t & 1;
      if (t >= 2 && !wait_all(PB_SEMPTY + b, ((t - 2) >> 1) & 1)) return false;
      if (!wait_all(PB_KFULL + s, (t / kPairKSlots) & 1)) return false;
      tc_fence_after();
      const uint64_t ka = dK + static_cast<uint64_t>((s * PairSmem::kTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        umma_f16_elect(tmem + kTmemS + 128u * b, dQ + off, ka + off, idS, kk > 0 ? 1u : 0u);
      }
      umma_commit_elect(bar(PB_SFULL + b));
      umma_commit_elect(bar(PB_KEMPTY + s));
      return true;
    };
    auto issue_pv = [&](int u) -> bool {
      const int sv = u % kPairVSlots, b = u & 1;
      if (!wait_all(PB_PFULL + b, (u >> 1) & 1)) return false;
      if (!wait_all(PB_VFULL + sv, (u / kPairVSlots) & 1)) return false;
      tc_fence_after();
      const uint64_t va = dV + static_cast<uint64_t>((sv * PairSmem::kTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        umma_ts_elect(tmem + kTmemO, tmem + kTmemP + 64u * b + 8u * kk, va + kk * 128, idO,
                      (u > 0 || kk > 0) ? 1u : 0u);
      umma_commit_elect(bar(PB_PVDONE + b));
      umma_commit_elect(bar(PB_VEMPTY + sv));
      return true;
    };
    bool ok = wait_all(PB_Q, 0);
    if (ok) ok = issue_s(0);
    if (ok && T > 1) ok = issue_s(1);
    for (int u = 0; ok && u < T; ++u) {
      if (__any_sync(0xffffffffu, *s_abort != 0)) { ok = false; break; }
      if (u + 2 < T && !issue_s(u + 2)) { ok = false; break; }
      if (!issue_pv(u)) { ok = false; break; }
    }
    if (!ok && lane == 0) *s_abort = 1;
    umma_commit_elect(bar(PB_DRAIN));
    mbar_wait(bar(PB_DRAIN), 0);
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ row-max warps
    const int q = warp;
    const int r = 32 * q + lane;
    const int side = r >> 6;                  // 0: rows of qa, 1: rows of qb (uniform per warp)
    const uint32_t lrow = static_cast<uint32_t>(32 * q) << 16;
    const float sc = prm.scale_log2;
    float m = -INFINITY;                      // running reference max (log2 units) of this row
    bool live = true;
    const float* orow = offset_row(side);
    float o0 = offset_of(orow, 0), o1 = offset_of(orow, 1);   // this tile's offsets, fetched a tile ahead
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      const float c0 = o0, c1 = o1;
      o0 = offset_of(orow, 2 * t + 2);
      o1 = offset_of(orow, 2 * t + 3);
      wait_live(bar(PB_SFULL + b), (t >> 1) & 1, live);
      tc_fence_after();
      const bool v0 = (s_union[2 * t] >> (16 + side)) & 1;
      const bool v1 = (2 * t + 1 < nu) && ((s_union[2 * t + 1] >> (16 + side)) & 1);
      float tmax = -INFINITY;                 // max over the tile's kept columns of x * scale + offset
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        if (hb == 0 ? v0 : v1) {
          uint32_t u[64];
          tmem_ld32(tmem + kTmemS + 128u * b + 64u * hb + lrow, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld32(tmem + kTmemS + 128u * b + 64u * hb + 32u + lrow, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_wait_ld();
          float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            m0 = fmax3(m0, __uint_as_float(u[c]), __uint_as_float(u[c + 1]));
            m1 = fmax3(m1, __uint_as_float(u[c + 2]), __uint_as_float(u[c + 3]));
          }
          const float hm = fmaxf(m0, m1) * sc;
          tmax = fmaxf(tmax, OFFSETS ? hm + (hb == 0 ? c0 : c1) : hm);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(PB_SEMPTY + b));
      float a = 1.0f;
      if (tmax > m + kPairRescale) {   // also the row's first kept tile (m = -inf)
        if (m != -INFINITY) a = fast_exp2(m - tmax);
        m = tmax;
      }
      // P buffer b is rewritten for tile t only after PV(t-2), its last reader, has completed.  The
      // exponential warps learn that from the reference-ready barrier, published after this wait.
      // The same wait keeps this warp (which runs ahead) from arriving on P full for tile t while
      // that barrier's phase still waits for the exponential warps' tile t-2.
      if (t >= 2) wait_live(bar(PB_PVDONE + b), ((t - 2) >> 1) & 1, live);
      s_ring[b * 128 + r] = make_float2(m, a);
      mbar_arrive(bar(PB_MREADY + 4 * b + q));
      if (__any_sync(0xffffffffu, a != 1.0f)) {
        // rescale these rows of O; PV(t-1), the last product into O, must be done
        wait_live(bar(PB_PVDONE + ((t - 1) & 1)), ((t - 1) >> 1) & 1, live);
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tmem + kTmemO + c0 + lrow, ov);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * a);
          tmem_st32(tmem + kTmemO + c0 + lrow, ov);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(PB_PFULL + b));
    }
  } else {
    // ------------------------------------------------------------ exponential warps
    const int q = warp & 3;                   // TMEM lane quarter
    const int hc = (warp - 4) >> 2;           // key block of the tile (S columns 64*hc ..)
    const int r = 32 * q + lane;              // query row in the 128-row tile
    const int side = r >> 6;                  // 0: qa, 1: qb
    const uint32_t lrow = static_cast<uint32_t>(32 * q) << 16;
    const float sc = prm.scale_log2;
    const float2 sc2 = make_float2(sc, sc);
    float m = -INFINITY;                      // this row's reference for the current tile
    float2 l2 = make_float2(0.0f, 0.0f);      // partial row sum of 2^(x - m) over this warp's columns
    float2 lb2 = make_float2(0.0f, 0.0f);     // the same sum over the bf16-rounded weights that enter P . V
    bool live = true;
    int ent = (hc < nu) ? s_union[hc] : 0;    // union entry of this warp's key block, one tile ahead
    const float* orow = offset_row(side);
    float offn = offset_of(orow, hc);         // its offset (log2 units), one tile ahead
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      const float offc = offn;
      offn = offset_of(orow, 2 * t + 2 + hc);
      wait_live(bar(PB_MREADY + 4 * b + q), (t >> 1) & 1, live);
      const float2 ma = s_ring[b * 128 + r];
      const bool vh = (2 * t + hc < nu) && ((ent >> (16 + side)) & 1);   // uniform per warp
      ent = (2 * t + 2 + hc < nu) ? s_union[2 * t + 2 + hc] : 0;
      m = ma.x;
      l2.x *= ma.y;
      l2.y *= ma.y;
      lb2.x *= ma.y;
      lb2.y *= ma.y;
      tc_fence_after();
      uint32_t u[64];
      if (vh) {
        tmem_ld32(tmem + kTmemS + 128u * b + 64u * hc + lrow, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld32(tmem + kTmemS + 128u * b + 64u * hc + 32u + lrow, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar(PB_SEMPTY + b));
      // P = 2^(x*scale - m) on kept columns, 0 elsewhere; bf16 pairs (keys 2c, 2c+1)
      uint32_t pk[32];
      if (vh) {
        const float2 nm = make_float2(offc - m, offc - m);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 x = ffma2(make_float2(__uint_as_float(u[2 * c]), __uint_as_float(u[2 * c + 1])), sc2, nm);
          const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          l2 = fadd2(l2, p);
          pk[c] = pack_bf16x2(p.x, p.y);
          lb2 = fadd2(lb2, make_float2(__uint_as_float(pk[c] << 16), __uint_as_float(pk[c] & 0xFFFF0000u)));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      // PV(t-2), the P buffer's last reader, completed before the reference for tile t was published
      tmem_st32(tmem + kTmemP + 64u * b + 32u * hc + lrow, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(PB_PFULL + b));
    }

    // ---- epilogue: O / l, bf16 store (this warp's half of the columns), log-sum-exp
    // o is normalised by the sum of the weights it was accumulated with (the bf16-rounded P), so a row
    // whose attention sits on one key errs only by o's own rounding; lse takes the float32 sum.
    const float lpart = l2.x + l2.y, lbpart = lb2.x + lb2.y;
    if (!mbar_wait(bar(PB_DRAIN), 0)) *s_abort = 1;   // every MMA of the CTA has completed
    tc_fence_after();
    s_lsum[hc * 128 + r] = lpart;
    s_lsum[256 + hc * 128 + r] = lbpart;
    named_bar_sync(1u + static_cast<uint32_t>(q), 64);
    const float lt = lpart + s_lsum[(hc ^ 1) * 128 + r];
    const float ltb = lbpart + s_lsum[256 + (hc ^ 1) * 128 + r];
    if (side == 0 || has_b) {
      const float inv = (ltb > 0.0f) ? 1.0f / ltb : 0.0f;
      const long long orow = out_row(side ? qb : qa, r & 63);
      uint4* dst = reinterpret_cast<uint4*>(prm.o + orow * D + (D / 2) * hc);
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32(tmem + kTmemO + (D / 2) * hc + c0 + lrow, ov);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * inv, __uint_as_float(ov[2 * c + 1]) * inv);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[c0 / 8 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
      if (prm.lse && hc == 0) prm.lse[orow] = (lt > 0.0f) ? (m + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dbst
