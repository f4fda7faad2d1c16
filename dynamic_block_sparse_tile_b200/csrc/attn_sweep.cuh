// Block-sparse attention kernels built on one tile walk: a CTA keeps its own 128 rows (two
// 64-token blocks) in shared memory while the 64-row blocks of the other side stream through a
// ring, one block per tile, over the union of the two own blocks' lists.  Uses:
//   MODE 0  backward, dq pass            MODE 1  backward, dk/dv pass
//   MODE 2  forward with 4-token group masks (and optional logit offsets)
//   MODE 3  forward over gathered 4-token key groups
//
// ---- Backward (MODES 0 and 1)
// The NABLA page ("NABLA: Neighborhood Adaptive Block-Level Attention",
// section "Contributions Clés", double-phase acceleration, and section
// "Résultats Expérimentaux", items 1 and 2: fine-tuning and pre-training) uses
// the same adaptive mask in training, which needs the gradient of the masked
// attention.  It is the exact
// gradient of the forward definition: for query block i with kept key tokens
// S_i, P = softmax(scale * q_i k_S^T), dP = dO_i v_S^T, delta = rowsum(P * dP)
// (one value per query row; it equals rowsum(dO_i * o_i)) and dS = P * (dP - delta):
//     dv_S += P^T dO_i,   dq_i = scale * dS k_S,   dk_S += scale * dS^T q_i.
// P is recomputed from the forward's log-sum-exp (P = 2^(s * scale * log2 e -
// lse * log2 e)), so no attention matrix is stored.
//
// delta is summed from the same float32 P and dP that form dS, not taken as
// dO . o from the forward's output: o is bf16, and where a row's attention sits on
// one key the true dq is close to zero while dO . (o_bf16 - o) is not, so that
// shortcut leaves a relative error of order 10 % in such rows' dq.  Summing P * dP
// keeps sum_j dS_ij = 0 to rounding, and the forward's o is not needed at all.
//
// Two launches:
//   sweep_kernel<..., 0>  dq: one CTA per pair of query blocks, over the union of their kept key
//                         blocks (the forward's lists), one key block per tile, in two sweeps:
//                         the first sums delta, the second forms dS and dq; it also writes
//                         (lse * log2 e, delta) of its rows to a tile-ordered stats array
//   sweep_kernel<..., 1>  dk, dv: one CTA per pair of key blocks, over the union of the query
//                         blocks that keep them (the transposed lists), one query block per tile
// Both passes have one shape.  The CTA's own 128 rows X, X2 (dq: Q, dO; dk/dv: K, V) stay in
// shared memory; per tile the 64 rows Y, Y2 of the other block (dq: K, V; dk/dv: Q, dO) arrive
// through a ring, and
//     A  = X . Y^T    [128 x 64]    (tcgen05 SS; dq: S, dk/dv: S^T)
//     A2 = X2 . Y2^T  [128 x 64]    (tcgen05 SS; dq: dP, dk/dv: dP^T)
// the softmax warps form P and dS from them in place in tensor memory (bf16 pairs), and
//     dq pass:    acc0 += dS . Y            (dq; tcgen05 TS, Y = K read MN-major)
//     dk/dv pass: acc0 += P^T . Y2          (dv; Y2 = dO)
//                 acc1 += dS^T . Y          (dk; Y = Q)
// A row (or column) whose block does not keep the tile's block gets P = dS = 0.
//
// ---- Forward with logit offsets and group masks (MODE 2)
// A forward for AB-Attention's finer selections ("AB-Attention accélère la génération vidéo…",
// section "Les trois techniques"): the 4-token key groups of the third technique (a 16-bit mask
// per (query block, key block) masks columns), with an optional logit offset per (query block,
// key block).  (SIP's offsets alone run in pair_attn_kernel, which folds them into its exponent.)
// One CTA per pair of query blocks
// (X = Q), the ring brings K and V (Y, Y2), two sweeps over the union: the first only forms
// S = Q K^T and keeps each row's running max and sum of 2^(x - max), x = s * scale * log2 e +
// offset * log2 e; the two column halves are merged into the row max M and L = log2 of the
// row's normaliser; the second sweep forms S again, P = 2^(x - M) as bf16 pairs in place, and
//     acc0 += P . Y2                      (o; tcgen05 TS, V read MN-major)
// and the epilogue scales o by 2^(M - L).  Relative to the final max, the largest weight of a
// row is exactly 1 in bf16 (as in pair_attn_kernel); normalising before the rounding instead
// costs about 0.006 of max-abs error where a row sits on one key.  No rescaling of o between
// tiles is needed.  Three 128x64xD products per tile against the two of pair_attn_kernel, for a
// kernel whose offsets cost nothing extra.  With a group mask (AB-Attention's third technique,
// key groups of 4 tokens), bit r of mask[i][j] keeps tokens 4r .. 4r+3 of key block j for query
// block i; the other columns get P = 0 in both sweeps.
//
// TMEM (512 columns): acc0 at 0, acc1 at 128, two tile buffers at 256 and 384; in buffer b the
// A product sits at +0 .. +63 and A2 at +64 .. +127.  Softmax warp (q, hc) reads columns
// 32hc .. 32hc+31 of both and writes its 32 bf16 results of each, packed in pairs, back into
// columns 32hc .. 32hc+15: inside the range it has itself read, so no other warp's input is
// overwritten.  The TS product over K = 64 then takes, for its 16-wide step kk, columns
// 32 * (kk >> 1) + 8 * (kk & 1) .. +7.
//
// Warp roles (320 threads):
//   warps 0-7  softmax warps: warp w covers TMEM lanes (rows) 32*(w%4) .. +31 and tile columns
//              32*(w/4) .. +31; then the epilogue of the same rows and half of the columns
//   warp 8     TMEM owner and MMA issuer (whole warp, one elected lane issues)
//   warp 9     TMA producer (lane 0): the own rows once, then the ring
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "attn_pair.cuh"
#include "ptx.cuh"
#include "reorder.cuh"

namespace dbst {

constexpr int kSweepThreads = 320;
constexpr int kSweepSlots = 3;

struct SweepParams {
  const int32_t* count;      // [BH*NB]: own block -> number of other blocks in its list
  const int16_t* idx;        // [BH*NB*NB]: the lists, ascending
  const float* lse;          // [BH*N] the forward's log-sum-exp, same layout as q (dq pass)
  float2* stats;             // [BH*N] tile order: (lse * log2 e, delta); written by the dq pass
  const float* offsets;      // MODE 2: [BH*NB*NB] natural-log offset of (query block, key block), or null
  const uint16_t* gmask;     // MODE 2: [BH*NB*NB] kept 4-token groups of (query block, key block), or null
  float* lse_out;            // MODE 2: [BH*N] log-sum-exp of the offset logits, same layout as q, or null
  __nv_bfloat16* out0;       // dq pass: dq; dk/dv pass: dv; MODE 2: o
  __nv_bfloat16* out1;       // dk/dv pass: dk
  int NB, N;
  int pair_stride;           // own blocks a and a + pair_stride share a CTA
  int pairs_per_head;
  float scale_log2;          // softmax scale * log2 e
  float scale;               // softmax scale
  long long wait_limit;      // cycles a wait between roles may take before the CTA gives up (0: default)
  TileGeo tg;                // token grid and tile shape (raster layout only)
};

// Shared-memory layout.  Modes 0-2 walk key (or query) blocks: at most 4096 union entries over
// 128 words of 32 blocks.  Mode 3 walks 4-token key groups, 16 per block: up to 16384 entries over
// 512 words, and it has no second own tile, so its ring starts right after X.
template <int MODE>
struct SweepLayout {
  static constexpr int kUnionCap = MODE == 3 ? 16384 : 4096;
  static constexpr int kMaxWords = kUnionCap / 32;
  static constexpr int kOwnX = 0;                         // X: D-halves x [128 rows x 128 B]
  static constexpr int kOwnX2 = 32768;                    // X2, same layout (modes 0 and 1)
  static constexpr int kRing = MODE == 3 ? 32768 : 65536;
  static constexpr int kSlot = 33792;                     // Y: D-halves x [64 rows x 128 B]; Y2 at +16384;
  static constexpr int kSlotY2 = 16384;                   //   64 float2 stats of Y's rows at +32768
  static constexpr int kSlotStats = 32768;
  static constexpr int kUnion = kRing + kSweepSlots * kSlot;   // int32 x kUnionCap: j | inA<<16 | inB<<17
  static constexpr int kWords = kUnion + 4 * kUnionCap;   // u32 [2][kMaxWords] bitmasks of the two lists
  static constexpr int kScan = kWords + 8 * kMaxWords;    // int [kMaxWords] word offsets
  static constexpr int kDelta = kScan + 4 * kMaxWords;    // float [2 quantities][2 column halves][128 rows]
  static constexpr int kBars = kDelta + 2048;
  static constexpr int kMisc = kBars + 256;
  static constexpr int kBytes = kMisc + 64;
  static_assert(kSlot % 1024 == 0 && kRing % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(kBytes + 1024 <= 227 * 1024, "shared memory per CTA");
};
using SweepSmem = SweepLayout<0>;
static_assert(SweepLayout<0>::kBytes == SweepLayout<1>::kBytes && SweepLayout<0>::kBytes == SweepLayout<2>::kBytes,
              "modes 0-2 share one layout");

enum {
  BB_OWN = 0,
  BB_RFULL = 1,                          // [kSweepSlots] ring slot loaded
  BB_REMPTY = BB_RFULL + kSweepSlots,      // [kSweepSlots] ring slot's last reader (the TS products) done
  BB_SFULL = BB_REMPTY + kSweepSlots,      // [2] A and A2 of tile t in buffer t&1 complete
  BB_PFULL = BB_SFULL + 2,               // [2] 256 arrivals: P / dS of tile t written
  BB_DRAIN = BB_PFULL + 2,
  BB_COUNT = BB_DRAIN + 1
};
static_assert(BB_COUNT * 8 <= 256, "barrier area");

constexpr uint32_t kSweepAcc0 = 0, kSweepAcc1 = 128, kSweepBuf = 256;

// 1-D bulk copy global -> shared, completing on `bar`; both addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// bits_t[bh][j][w] bit i = bits[bh][32w + i][j / 32] bit (j % 32): key block j's row lists the
// query blocks whose kept set contains j.
__global__ void __launch_bounds__(256) transpose_bits_kernel(const uint32_t* __restrict__ bits,
                                                             uint32_t* __restrict__ bits_t, int NB, int NW,
                                                             long long words) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < words; e += stride) {
    const long long bh = e / (static_cast<long long>(NB) * NW);
    const int rem = static_cast<int>(e - bh * NB * NW);
    const int j = rem / NW, w = rem % NW;
    const uint32_t* head = bits + bh * NB * NW;
    uint32_t word = 0u;
    for (int i = 0; i < 32; ++i) {
      const int qi = 32 * w + i;
      if (qi >= NB) break;
      word |= ((head[static_cast<long long>(qi) * NW + (j >> 5)] >> (j & 31)) & 1u) << i;
    }
    bits_t[e] = word;
  }
}

// MODE 0: dq pass (X = Q, X2 = dO, Y = K, Y2 = V; lists = the forward's kept key blocks);
//         virtual tiles v = 0 .. 2T-1 walk the union twice (tile v mod T).
// MODE 1: dk/dv pass (X = K, X2 = V, Y = Q, Y2 = dO; lists = the transposed lists), T tiles.
// MODE 2: forward with offsets (X = Q, Y = K, Y2 = V; the forward's lists), 2T virtual tiles; X2
//         is not used, and the first sweep loads only Y.
// RASTER: tensors in the caller's raster order, loaded with 5-D boxes (see pair_attn_kernel).
template <int D, bool RASTER, int MODE>
__global__ void __launch_bounds__(kSweepThreads, 1)
    sweep_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmX2,
               const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmY2,
               const SweepParams prm) {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(MODE >= 0 && MODE <= 3, "mode");
  using L = SweepLayout<MODE>;
  constexpr bool DKDV = MODE == 1;
  constexpr bool GATHER = MODE == 3;            // the forward over gathered 4-token key groups
  constexpr bool FWD = MODE == 2 || GATHER;     // the forward sweeps (offsets, group masks, gather)
  constexpr int DH = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  int32_t* s_union = reinterpret_cast<int32_t*>(sm + L::kUnion);
  uint32_t* s_words = reinterpret_cast<uint32_t*>(sm + L::kWords);
  int32_t* s_scan = reinterpret_cast<int32_t*>(sm + L::kScan);
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(sm + L::kMisc);
  volatile uint32_t* s_abort = s_misc + 2;
  auto bar = [&](int slot) -> uint32_t { return sbase + L::kBars + 8u * slot; };
  // waits between roles run out after `limit` cycles; the drains of a CTA's own copies and
  // products keep the default limit
  const long long limit = prm.wait_limit > 0 ? prm.wait_limit : kWaitLimitCycles;
  auto wait_live = [&](uint32_t mb, uint32_t parity, bool& live) {
    if (!live || mbar_try(mb, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try(mb, parity)) {
      if (*s_abort) { live = false; return; }
      if (clock64() - t0 > limit) {
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
  const int ps = prm.pair_stride;
  const int ba = (pi / ps) * 2 * ps + (pi % ps);
  const int bb = ba + ps;
  const bool has_b = bb < NB;
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
  // Mode 3: TMA load of 4-token group grp's channels 64h .. 64h+63 (4 rows, 512 B); the map's box
  // is 4 rows high (RASTER: 4 tokens along x, which the host requires tx to allow)
  auto load_group = [&](uint32_t dst, const CUtensorMap* map, uint32_t mbar, int grp, int h) {
    if constexpr (RASTER) {
      const int blk = grp >> 4, off = (grp & 15) * 4;
      const int Tx = blk % prm.tg.nX, Ty = (blk / prm.tg.nX) % prm.tg.nY, Tt = blk / (prm.tg.nX * prm.tg.nY);
      const int dx = off % prm.tg.tx, dy = (off / prm.tg.tx) % prm.tg.ty, dt = off / (prm.tg.tx * prm.tg.ty);
      tma_load_5d(dst, map, mbar, 64 * h, Tx * prm.tg.tx + dx, Ty * prm.tg.ty + dy, Tt * prm.tg.tt + dt,
                  static_cast<int32_t>(bh));
    } else {
      tma_load_2d(dst, map, mbar, 64 * h, static_cast<int32_t>(bh * prm.N + static_cast<long long>(grp) * 4));
    }
  };

  for (int w = tid; w < 2 * L::kMaxWords; w += kSweepThreads) s_words[w] = 0u;
  if (tid == 0) {
    for (int b = 0; b < BB_COUNT; ++b) mbar_init(bar(b), (b == BB_PFULL || b == BB_PFULL + 1) ? 256u : 1u);
    fence_mbar_init();
    for (int i = 1; i < 16; ++i) s_misc[i] = 0;
  }
  __syncthreads();
  if (warp == 9 && lane == 0) {   // own rows: blocks ba (rows 0..63) and bb (rows 64..127; ba again if none)
    tma_prefetch_desc(&tmX);
    if constexpr (!FWD) tma_prefetch_desc(&tmX2);
    mbar_expect_tx(bar(BB_OWN), (FWD ? 1 : 2) * 128 * D * 2);
    for (int h = 0; h < DH; ++h) {
      load_block(sbase + L::kOwnX + h * 16384, &tmX, bar(BB_OWN), ba, h);
      load_block(sbase + L::kOwnX + h * 16384 + 8192, &tmX, bar(BB_OWN), has_b ? bb : ba, h);
      if constexpr (!FWD) {
        load_block(sbase + L::kOwnX2 + h * 16384, &tmX2, bar(BB_OWN), ba, h);
        load_block(sbase + L::kOwnX2 + h * 16384 + 8192, &tmX2, bar(BB_OWN), has_b ? bb : ba, h);
      }
    }
  }
  if (warp == 8) {
    tmem_alloc(sbase + L::kMisc, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  // ---- union of the two own blocks' lists -> ascending entries with membership flags
  // (mode 3: of their kept 4-token groups, read from the group masks: word w holds blocks 2w, 2w+1)
  const int NWu = GATHER ? (16 * NB + 31) >> 5 : NW;
  if constexpr (GATHER) {
    const uint16_t* m0 = prm.gmask + (bh * NB + ba) * static_cast<long long>(NB);
    const uint16_t* m1 = prm.gmask + (bh * NB + (has_b ? bb : ba)) * static_cast<long long>(NB);
    for (int e = tid; e < 2 * NWu; e += kSweepThreads) {
      const int side = e >= NWu;
      const int w = side ? e - NWu : e;
      if (side && !has_b) continue;
      const uint16_t* m = side ? m1 : m0;
      const uint32_t lo = m[2 * w], hi = (2 * w + 1 < NB) ? m[2 * w + 1] : 0u;
      s_words[side * L::kMaxWords + w] = lo | (hi << 16);
    }
  } else {
  int n0 = prm.count[bh * NB + ba];
  int n1 = has_b ? prm.count[bh * NB + bb] : 0;
  if (n0 < 0 || n0 > NB || n1 < 0 || n1 > NB) {
    if (tid == 0) record_error(kErrBounds);
    n0 = min(max(n0, 0), NB);
    n1 = min(max(n1, 0), NB);
  }
  const int16_t* g0 = prm.idx + (bh * NB + ba) * static_cast<long long>(NB);
  const int16_t* g1 = prm.idx + (bh * NB + (has_b ? bb : ba)) * static_cast<long long>(NB);
  for (int e = tid; e < n0 + n1; e += kSweepThreads) {
    const int side = e >= n0;
    const int j = static_cast<int>(side ? g1[e - n0] : g0[e]);
    if (j < 0 || j >= NB) {
      record_error(kErrBounds);
      continue;
    }
    atomicOr(&s_words[side * L::kMaxWords + (j >> 5)], 1u << (j & 31));
  }
  }
  __syncthreads();
  if (warp == 0) {   // exclusive scan of the union's popcounts over NWu <= kMaxWords words
    constexpr int WPL = L::kMaxWords / 32;
    int cnt[WPL], tot = 0;
#pragma unroll
    for (int e = 0; e < WPL; ++e) {
      const int w = WPL * lane + e;
      cnt[e] = (w < NWu) ? __popc(s_words[w] | s_words[L::kMaxWords + w]) : 0;
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
    for (int e = 0; e < WPL; ++e) {
      s_scan[WPL * lane + e] = run;
      run += cnt[e];
    }
    if (lane == 31) s_misc[1] = static_cast<uint32_t>(incl);
  }
  __syncthreads();
  for (int w = tid; w < NWu; w += kSweepThreads) {
    const uint32_t wa = s_words[w], wb = s_words[L::kMaxWords + w];
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
  const int nu = static_cast<int>(s_misc[1]);   // union entries (blocks; mode 3: groups)
  const int T = GATHER ? (nu + 15) >> 4 : nu;   // tiles: one block, or 16 groups
  const int NV = DKDV ? T : 2 * T;       // virtual tiles
  const int v_ts = DKDV ? 0 : T;         // first virtual tile with TS products
  if (T == 0) {   // nothing in either list: zero gradients; MODE 2: o = 0 and lse = -inf
    if (warp == 9 && lane == 0) mbar_wait(bar(BB_OWN), 0);
    if (warp == 8) tmem_dealloc(tmem, 512);
    for (int e = tid; e < 64 * D / 8; e += kSweepThreads) {
      const int rr = e / (D / 8), c = e % (D / 8);
      const uint4 z = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(prm.out0 + out_row(ba, rr) * D)[c] = z;
      if (has_b) reinterpret_cast<uint4*>(prm.out0 + out_row(bb, rr) * D)[c] = z;
      if constexpr (DKDV) {
        reinterpret_cast<uint4*>(prm.out1 + out_row(ba, rr) * D)[c] = z;
        if (has_b) reinterpret_cast<uint4*>(prm.out1 + out_row(bb, rr) * D)[c] = z;
      }
    }
    if constexpr (FWD) {
      if (prm.lse_out && tid < 64) {
        prm.lse_out[out_row(ba, tid)] = -INFINITY;
        if (has_b) prm.lse_out[out_row(bb, tid)] = -INFINITY;
      }
    }
    return;
  }

  if (warp == 9 && GATHER) {
    // ------------------------------------------------------------ mode 3 producer: 16 groups per tile
    // Lane 0 waits for the slot and arms its barrier; then lanes 0-15 each load one group (the
    // first group of the tile stands in past the end of the union; its columns are masked).
    if (lane == 0) {
      tma_prefetch_desc(&tmY);
      tma_prefetch_desc(&tmY2);
    }
    int armed[kSweepSlots] = {0, 0, 0};
    for (int v = 0; v < NV; ++v) {
      const int s = v % kSweepSlots;
      int ok = 1;
      if (lane == 0) {
        if (*s_abort) {
          ok = 0;
        } else if (v >= kSweepSlots && !mbar_wait_lim(bar(BB_REMPTY + s), ((v / kSweepSlots) - 1) & 1, limit)) {
          *s_abort = 1;
          ok = 0;
        } else {
          mbar_expect_tx(bar(BB_RFULL + s), (v >= T ? 2 : 1) * 64 * D * 2);   // values in the second sweep
          armed[s] = v / kSweepSlots + 1;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();
      if (lane < 16) {
        const int t = v < T ? v : v - T;
        const int u = 16 * t + lane;
        const int grp = (u < nu ? s_union[u] : s_union[16 * t]) & 0xFFFF;
        const uint32_t dst = sbase + L::kRing + s * L::kSlot + 512u * lane;
        for (int h = 0; h < DH; ++h) {
          load_group(dst + h * 8192, &tmY, bar(BB_RFULL + s), grp, h);
          if (v >= T) load_group(dst + L::kSlotY2 + h * 8192, &tmY2, bar(BB_RFULL + s), grp, h);
        }
      }
    }
    if (lane == 0) {   // no copy may still be landing when the CTA exits
      for (int s = 0; s < kSweepSlots; ++s)
        if (armed[s] > 0) mbar_wait(bar(BB_RFULL + s), (armed[s] - 1) & 1);
      mbar_wait(bar(BB_OWN), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ TMA producer of the ring
    if (lane == 0) {
      tma_prefetch_desc(&tmY);
      tma_prefetch_desc(&tmY2);
      int armed[kSweepSlots] = {0, 0, 0};
      for (int t = 0; t < NV; ++t) {
        if (*s_abort) break;
        const int s = t % kSweepSlots;
        if (t >= kSweepSlots && !mbar_wait_lim(bar(BB_REMPTY + s), ((t / kSweepSlots) - 1) & 1, limit)) {
          *s_abort = 1;
          break;
        }
        const int j = s_union[t < T ? t : t - T] & 0xFFFF;
        const uint32_t dst = sbase + L::kRing + s * L::kSlot;
        const bool withY2 = !(FWD && t < T);   // the offset forward's first sweep needs no values
        mbar_expect_tx(bar(BB_RFULL + s), (withY2 ? 2 : 1) * 64 * D * 2 + (DKDV ? 512 : 0));
        for (int h = 0; h < DH; ++h) {
          load_block(dst + h * 8192, &tmY, bar(BB_RFULL + s), j, h);
          if (withY2) load_block(dst + L::kSlotY2 + h * 8192, &tmY2, bar(BB_RFULL + s), j, h);
        }
        if constexpr (DKDV)
          bulk_load_1d(dst + L::kSlotStats, prm.stats + bh * prm.N + static_cast<long long>(j) * 64, 512,
                       bar(BB_RFULL + s));
        armed[s] = t / kSweepSlots + 1;
      }
      // no copy may still be landing when the CTA exits
      for (int s = 0; s < kSweepSlots; ++s)
        if (armed[s] > 0) mbar_wait(bar(BB_RFULL + s), (armed[s] - 1) & 1);
      mbar_wait(bar(BB_OWN), 0);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    constexpr uint32_t idSS = idesc_bf16(128, 64, 0, 0);   // A = own rows (K-major), B = ring rows (K-major)
    constexpr uint32_t idTS = idesc_bf16(128, D, 0, 1);    // A = P or dS in TMEM, B = ring rows (MN-major)
    const uint64_t dX = smem_desc(sbase + L::kOwnX, 16, 1024);
    const uint64_t dX2 = smem_desc(sbase + L::kOwnX2, 16, 1024);
    const uint64_t dRingK = smem_desc(sbase + L::kRing, 16, 1024);
    const uint64_t dRingMN = smem_desc(sbase + L::kRing, 8192, 1024);
    auto wait_all = [&](int slot, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_lim(bar(slot), parity, limit));
    };
    auto issue_ss = [&](int t) -> bool {
      const int s = t % kSweepSlots, b = t & 1;
      if (!wait_all(BB_RFULL + s, (t / kSweepSlots) & 1)) return false;
      tc_fence_after();
      const uint64_t y = dRingK + static_cast<uint64_t>((s * L::kSlot) >> 4);
      const uint64_t y2 = y + static_cast<uint64_t>(L::kSlotY2 >> 4);
      const uint32_t acc = tmem + kSweepBuf + 128u * b;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t oa = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        const uint32_t ob = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
        umma_f16_elect(acc, dX + oa, y + ob, idSS, kk > 0 ? 1u : 0u);
        if constexpr (!FWD) umma_f16_elect(acc + 64u, dX2 + oa, y2 + ob, idSS, kk > 0 ? 1u : 0u);
      }
      umma_commit_elect(bar(BB_SFULL + b));
      return true;
    };
    // Virtual tile u: once the softmax warps are done with buffer u&1, the TS products (second
    // sweep of the dq pass, every tile of the dk/dv pass); the commits then also mark the buffer
    // and the ring slot free in the first sweep, which has no TS products.
    auto issue_ts = [&](int u) -> bool {
      const int s = u % kSweepSlots, b = u & 1;
      if (!wait_all(BB_PFULL + b, (u >> 1) & 1)) return false;
      tc_fence_after();
      const uint64_t y = dRingMN + static_cast<uint64_t>((s * L::kSlot) >> 4);
      const uint64_t y2 = y + static_cast<uint64_t>(L::kSlotY2 >> 4);
      const uint32_t buf = tmem + kSweepBuf + 128u * b;
      if (u >= v_ts) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t col = 32u * (kk >> 1) + 8u * (kk & 1);
          const uint32_t accf = (u > v_ts || kk > 0) ? 1u : 0u;
          if constexpr (DKDV) {
            umma_ts_elect(tmem + kSweepAcc0, buf + col, y2 + kk * 128, idTS, accf);          // dv += P^T dO
            umma_ts_elect(tmem + kSweepAcc1, buf + 64u + col, y + kk * 128, idTS, accf);     // dk += dS^T Q
          } else if constexpr (FWD) {
            umma_ts_elect(tmem + kSweepAcc0, buf + col, y2 + kk * 128, idTS, accf);          // o += P V
          } else {
            umma_ts_elect(tmem + kSweepAcc0, buf + 64u + col, y + kk * 128, idTS, accf);     // dq += dS K
          }
        }
      }
      umma_commit_elect(bar(BB_REMPTY + s));
      return true;
    };
    bool ok = wait_all(BB_OWN, 0);
    if (ok) ok = issue_ss(0);
    if (ok && NV > 1) ok = issue_ss(1);
    for (int u = 0; ok && u < NV; ++u) {
      if (__any_sync(0xffffffffu, *s_abort != 0)) { ok = false; break; }
      if (!issue_ts(u)) { ok = false; break; }
      // The products of tile u+2 rewrite buffer u&1, which the TS products of tile u read (P and dS):
      // tcgen05.mma operations issued by one thread execute in issue order, so they are queued right
      // behind them, with no wait for their completion.
      if (u + 2 < NV && !issue_ss(u + 2)) { ok = false; break; }
    }
    if (!ok && lane == 0) *s_abort = 1;
    umma_commit_elect(bar(BB_DRAIN));
    mbar_wait(bar(BB_DRAIN), 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int q = warp & 3;                   // TMEM lane quarter
    const int hc = warp >> 2;                 // tile columns 32hc .. 32hc+31
    const int r = 32 * q + lane;              // own row in the 128-row tile
    const int side = r >> 6;                  // 0: block ba, 1: block bb (uniform per warp)
    const uint32_t lrow = static_cast<uint32_t>(32 * q) << 16;
    const float sc = prm.scale_log2;
    float* s_delta = reinterpret_cast<float*>(sm + L::kDelta);
    if constexpr (FWD) {
      // ---- forward with offsets: first sweep row max and sum, second sweep P = 2^(x - M) and o += P V
      const int own = side ? bb : ba;
      const float* offrow = prm.offsets ? prm.offsets + (bh * NB + own) * static_cast<long long>(NB) : nullptr;
      const uint16_t* gmrow = prm.gmask ? prm.gmask + (bh * NB + own) * static_cast<long long>(NB) : nullptr;
      float m = -INFINITY, l = 0.0f;          // first sweep, this warp's columns: running max of x, sum of 2^(x - m)
      float M = -INFINITY, L = -INFINITY;     // the row's max of x and log2 of its normaliser
      bool live = true;
      for (int v = 0; v < NV; ++v) {
        const int b = v & 1;
        const int t = v < T ? v : v - T;
        wait_live(bar(BB_SFULL + b), (v >> 1) & 1, live);
        tc_fence_after();
        // this warp's 32 columns are the groups 8hc .. 8hc+7 of the tile: of the tile's key block,
        // or (mode 3) union entries 16t + 8hc .. +7
        uint32_t gbits = 0u;
        float off = 0.0f;
        if constexpr (GATHER) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int u = 16 * t + 8 * hc + e;
            if (u < nu && ((s_union[u] >> (16 + side)) & 1)) gbits |= 1u << e;
          }
        } else {
          const int ent = s_union[t];
          gbits = (((ent >> (16 + side)) & 1) == 0) ? 0u
                  : (gmrow != nullptr) ? ((gmrow[ent & 0xFFFF] >> (8 * hc)) & 0xFFu) : 0xFFu;
          if (gbits != 0u && offrow != nullptr) off = offrow[ent & 0xFFFF] * 1.4426950408889634f;
        }
        const bool vh = gbits != 0u;                 // uniform per warp
        const uint32_t buf = tmem + kSweepBuf + 128u * b + 32u * hc + lrow;
        if (v < T) {
          if (vh) {
            uint32_t sv[32];
            tmem_ld32(buf, sv);
            tmem_wait_ld();
            float smax = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if ((gbits >> (c >> 2)) & 1u) smax = fmaxf(smax, __uint_as_float(sv[c]));
            const float mn = fmaxf(m, fmaf(smax, sc, off));   // finite: a kept group is here
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if ((gbits >> (c >> 2)) & 1u) acc += fast_exp2(fmaf(__uint_as_float(sv[c]), sc, off - mn));
            l = fmaf(l, fast_exp2(m - mn), acc);               // m = -inf: 2^-inf = 0
            m = mn;
          }
          tc_fence_before();
          mbar_arrive(bar(BB_PFULL + b));
          if (v == T - 1) {   // merge the two column halves of each row
            s_delta[hc * 128 + r] = m;
            s_delta[256 + hc * 128 + r] = l;
            named_bar_sync(1u + static_cast<uint32_t>(q), 64);
            const float m0 = s_delta[r], m1 = s_delta[128 + r];
            M = fmaxf(m0, m1);
            if (M != -INFINITY)
              L = M + __log2f(s_delta[256 + r] * fast_exp2(m0 - M) + s_delta[384 + r] * fast_exp2(m1 - M));
          }
          continue;
        }
        uint32_t pp[16];
        if (vh) {
          uint32_t sv[32];
          tmem_ld32(buf, sv);
          tmem_wait_ld();
          const float nb = off - M;
#pragma unroll
          for (int c = 0; c < 16; ++c) {   // columns 2c and 2c+1 share group c/2
            const bool keep = (gbits >> (c >> 1)) & 1u;
            pp[c] = keep ? pack_bf16x2(fast_exp2(fmaf(__uint_as_float(sv[2 * c]), sc, nb)),
                                       fast_exp2(fmaf(__uint_as_float(sv[2 * c + 1]), sc, nb)))
                         : 0u;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) pp[c] = 0u;
        }
        tmem_st16(buf, pp);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(BB_PFULL + b));
      }
      // ---- epilogue: o = acc * 2^(M - L); this warp's rows, columns (D/2)hc .. +D/2
      if (!mbar_wait(bar(BB_DRAIN), 0)) *s_abort = 1;   // every MMA of the CTA has completed
      tc_fence_after();
      if (side == 0 || has_b) {
        const long long orow = out_row(own, r & 63);
        const float f = (L == -INFINITY) ? 0.0f : fast_exp2(M - L);
        uint4* dst = reinterpret_cast<uint4*>(prm.out0 + orow * D + (D / 2) * hc);
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tmem + kSweepAcc0 + (D / 2) * hc + c0 + lrow, ov);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * f, __uint_as_float(ov[2 * c + 1]) * f);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[c0 / 8 + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        if (hc == 0 && prm.lse_out != nullptr)
          prm.lse_out[orow] = (L == -INFINITY) ? -INFINITY : L * 0.69314718055994530942f;
      }
    } else {
      float rowL = 0.0f, rowD = 0.0f;           // dq pass: this query row's (lse * log2 e, delta)
      if constexpr (!DKDV) {
        if (side == 0 || has_b) rowL = prm.lse[out_row(side ? bb : ba, r & 63)] * 1.4426950408889634f;
      }
      bool live = true;
      float dsum = 0.0f;                        // dq pass, first sweep: sum of P * dP over this warp's columns
      for (int v = 0; v < NV; ++v) {
        const int b = v & 1, s = v % kSweepSlots;
        const int t = v < T ? v : v - T;
        wait_live(bar(BB_SFULL + b), (v >> 1) & 1, live);
        // the ring slot cannot be refilled before this tile's TS products, which wait for this warp
        if constexpr (DKDV) wait_live(bar(BB_RFULL + s), (v / kSweepSlots) & 1, live);
        tc_fence_after();
        const bool vh = (s_union[t] >> (16 + side)) & 1;   // uniform per warp
        const uint32_t buf = tmem + kSweepBuf + 128u * b + 32u * hc + lrow;
        if (v < v_ts) {   // dq pass, first sweep: delta only
          if (vh) {
            uint32_t sv[32], dv[32];
            tmem_ld32(buf, sv);
            tmem_ld32(buf + 64u, dv);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
              dsum = fmaf(fast_exp2(fmaf(__uint_as_float(sv[c]), sc, -rowL)), __uint_as_float(dv[c]), dsum);
          }
          tc_fence_before();
          mbar_arrive(bar(BB_PFULL + b));
          if (v == v_ts - 1) {   // combine the two column halves; publish (L, delta) for the dk/dv pass
            s_delta[hc * 128 + r] = dsum;
            named_bar_sync(1u + static_cast<uint32_t>(q), 64);
            rowD = s_delta[r] + s_delta[128 + r];
            if (hc == 0 && (side == 0 || has_b))
              prm.stats[bh * prm.N + static_cast<long long>(side ? bb : ba) * 64 + (r & 63)] = make_float2(rowL, rowD);
          }
          continue;
        }
        uint32_t pp[16], pd[16];
        if (vh) {
          uint32_t sv[32], dv[32];
          tmem_ld32(buf, sv);
          tmem_ld32(buf + 64u, dv);
          tmem_wait_ld();
          if constexpr (DKDV) {
            // column c of the tile is query row c of the ring block: (lse * log2 e, delta) per column
            const float4* st4 = reinterpret_cast<const float4*>(sm + L::kRing + s * L::kSlot +
                                                                L::kSlotStats) + 16 * hc;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float4 st = st4[c];
              const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * c]), sc, -st.x));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * c + 1]), sc, -st.z));
              const float d0 = p0 * (__uint_as_float(dv[2 * c]) - st.y);
              const float d1 = p1 * (__uint_as_float(dv[2 * c + 1]) - st.w);
              pp[c] = pack_bf16x2(p0, p1);
              pd[c] = pack_bf16x2(d0, d1);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * c]), sc, -rowL));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * c + 1]), sc, -rowL));
              pd[c] = pack_bf16x2(p0 * (__uint_as_float(dv[2 * c]) - rowD), p1 * (__uint_as_float(dv[2 * c + 1]) - rowD));
              pp[c] = 0u;
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) pp[c] = pd[c] = 0u;
        }
        if constexpr (DKDV) tmem_st16(buf, pp);
        tmem_st16(buf + 64u, pd);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(BB_PFULL + b));
      }

      // ---- epilogue: this warp's rows, columns (D/2)hc .. +D/2 of each accumulator, to bf16
      if (!mbar_wait(bar(BB_DRAIN), 0)) *s_abort = 1;   // every MMA of the CTA has completed
      tc_fence_after();
      if (side == 0 || has_b) {
        const long long orow = out_row(side ? bb : ba, r & 63);
        auto store = [&](uint32_t acc, __nv_bfloat16* out, float f) {
          uint4* dst = reinterpret_cast<uint4*>(out + orow * D + (D / 2) * hc);
#pragma unroll
          for (int c0 = 0; c0 < D / 2; c0 += 32) {
            uint32_t ov[32];
            tmem_ld32(tmem + acc + (D / 2) * hc + c0 + lrow, ov);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
              pk[c] = pack_bf16x2(__uint_as_float(ov[2 * c]) * f, __uint_as_float(ov[2 * c + 1]) * f);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[c0 / 8 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        };
        if constexpr (DKDV) {
          store(kSweepAcc0, prm.out0, 1.0f);        // dv
          store(kSweepAcc1, prm.out1, prm.scale);   // dk
        } else {
          store(kSweepAcc0, prm.out0, prm.scale);   // dq
        }
      }
      tc_fence_before();
    }
  }

  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dbst
