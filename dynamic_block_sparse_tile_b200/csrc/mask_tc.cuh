// Adaptive block mask with the pooled logits on the tensor cores (NABLA page,
// "Construction de Masque Adaptatif": block mean-pool, reduced attention map,
// CDF threshold; "Intégration Hybride avec STA": the sliding-tile union).
//
// Five kernels:
//
//   pool_pieces_kernel (HBM-bound) averages every 64-token block of q and k
//   exactly (64 bf16 values summed in float64) and stores each mean x as three
//   bf16 pieces b1 + b2 + b3 (round to nearest, each piece the rounded
//   remainder of the previous ones, together the float32 value of x) plus the
//   float32 residual x - (b1 + b2 + b3), and the block's norm.
//
//   pooled_logits_tc_kernel (persistent) takes items of R consecutive query
//   blocks of one head.  tcgen05 computes the pooled logits of the R rows
//   against every key block as S^T = Kp . Qp^T (M = 128 key blocks per tile,
//   N = R rows), from the pieces: D1 = b1 b1 and D2 = b1 b2 + b2 b1 + b1 b3 +
//   b2 b2 + b3 b1 in two fp32 accumulators; s = (D1 + D2) * scale goes to a
//   float32 map in the workspace (small enough to stay in L2 for the next
//   kernel).
//
//   select_rows_kernel, one warp per row and many rows in flight per SM, finds
//   the CDF boundary by bisection on the logit value with exact integer mass
//   sums (one warp reduction per step) and writes bits and lists, or lists the
//   row when another block lies within the error band of its boundary (below).
//
//   refine_rows_kernel settles the listed rows whose band fits a warp (float64
//   logits of the band's blocks, a shuffle sort), and refine_wide_kernel the rest
//   (a band widened until the crossing stays inside, radix select on exact keys).
//
// Exactness.  The order of a row's blocks must be the order of the exact
// (float64) logits.  The fast logits carry an error below E = 2^-15 * scale *
// |Qp_i| * max_j |Kp_j| (Cauchy-Schwarz on the neglected piece products, the
// representation errors and eight fp32 accumulation steps of D1, with a margin
// of four).  After the fast selection, every key whose fast logit lies within
// 4E of the boundary key's is recomputed exactly in float64 from the pieces and
// residuals, and the selection is repeated with those keys ordered exactly and
// all other keys placed above or below the band.  The result stands if the new
// boundary lies within 2E of the old one; otherwise the band doubles and the
// step repeats.  Masses are float32 exponentials of the fast logits, rounded to
// integers of 2^-21 (2^-20 for rows of more than 1024 blocks) of the row's
// largest and summed exactly; a kept set can therefore differ from a float64
// reference only where a cumulative mass lies within rounding of p.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "mask.cuh"
#include "ptx.cuh"
#include "reorder.cuh"

namespace dbst {

// ---------------------------------------------------------------------------
// Workspace of the tensor-core mask build (all offsets 256-byte aligned).
// ---------------------------------------------------------------------------
struct MaskTcBuffers {
  unsigned int* kmax;       // [BH] float bits of max_j |Kp_j| (zeroed before the pool kernel)
  __nv_bfloat16* pieces;    // [6][BH][NB][D]: q pieces 1..3, then k pieces 1..3
  float* resid;             // [2][BH][NB][D]: q, k residuals
  float* norm;              // [2][BH][NB]: q, k block norms (rounded up)
};

constexpr int kPoolTcThreads = 256;

template <int D, bool RASTER>
__global__ void __launch_bounds__(kPoolTcThreads) pool_pieces_kernel(const uint4* __restrict__ q,
                                                                     const uint4* __restrict__ k, MaskTcBuffers wb,
                                                                     long long BH, int NB, TileGeo tg) {
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
  const long long total = 2 * BH * NB;   // the q blocks of a head, then its k blocks
  const long long plane = BH * NB * static_cast<long long>(D);
  for (long long w = warp; w < total; w += nwarps) {
    const long long bh = w / (2 * NB);
    const int rem = static_cast<int>(w - bh * 2 * NB);
    const bool isk = rem >= NB;
    const int blk = isk ? rem - NB : rem;
    const uint4* src = (isk ? k : q) +
                       (bh * tg.N + (RASTER ? tiled_to_raster(blk * 64, tg) : static_cast<long long>(blk) * 64)) * CPR;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 8
    for (int r = r0; r < 64; r += RPW) {
      const uint4 v = ld_stream(src + (RASTER ? row_off[r] : r) * CPR + ch);
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
    // every lane now holds the sums of channels 8ch .. 8ch+7
    uint32_t pw[3][4];
    float res[8];
    double n2 = 0.0;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      uint32_t pr[3] = {0u, 0u, 0u};
#pragma unroll
      for (int f = 0; f < 2; ++f) {
        const double x = acc[e + f] * (1.0 / 64.0);
        n2 = fma(x, x, n2);
        const float hi = __double2float_rn(x);
        const __nv_bfloat16 b1 = __float2bfloat16_rn(hi);
        const float r1 = hi - __bfloat162float(b1);
        const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(b2);
        const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
        const double rep = static_cast<double>(__bfloat162float(b1)) + static_cast<double>(__bfloat162float(b2)) +
                           static_cast<double>(__bfloat162float(b3));
        res[e + f] = __double2float_rn(x - rep);
        pr[0] |= static_cast<uint32_t>(__bfloat16_as_ushort(b1)) << (16 * f);
        pr[1] |= static_cast<uint32_t>(__bfloat16_as_ushort(b2)) << (16 * f);
        pr[2] |= static_cast<uint32_t>(__bfloat16_as_ushort(b3)) << (16 * f);
      }
      pw[0][e / 2] = pr[0];
      pw[1][e / 2] = pr[1];
      pw[2][e / 2] = pr[2];
    }
#pragma unroll
    for (int off = 1; off < CPR; off <<= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, off);
    const long long row = (bh * NB + blk) * static_cast<long long>(D);
    if (r0 == 0) {
#pragma unroll
      for (int pc = 0; pc < 3; ++pc) {
        uint4* dst = reinterpret_cast<uint4*>(wb.pieces + (isk ? 3 + pc : pc) * plane + row + ch * 8);
        *dst = make_uint4(pw[pc][0], pw[pc][1], pw[pc][2], pw[pc][3]);
      }
      float4* rd = reinterpret_cast<float4*>(wb.resid + (isk ? plane : 0) + row + ch * 8);
      rd[0] = make_float4(res[0], res[1], res[2], res[3]);
      rd[1] = make_float4(res[4], res[5], res[6], res[7]);
    }
    if (lane == 0) {
      const float nrm = __double2float_ru(__dsqrt_ru(n2));
      wb.norm[(isk ? BH * NB : 0) + bh * NB + blk] = nrm;
      if (isk) atomicMax(wb.kmax + bh, __float_as_uint(nrm));   // non-negative floats order as their bits
    }
  }
}

// ---------------------------------------------------------------------------
// Selection kernel.
// ---------------------------------------------------------------------------
constexpr int kLogTcThreads = 192;       // warp 0 TMA, warp 1 MMA, warps 2..5 drain
constexpr int kLogTcDrain = 4;
constexpr int kLogTcStages = 3;          // K ring: one piece of one 64-channel half of one key tile

struct LogTcParams {
  MaskTcBuffers wb;
  float* S;            // out: [BH][NB][NB] fast pooled logits, already scaled
  long long BH;
  int NB;
  int ntiles;          // key tiles of 128 blocks: ceil(NB / 128)
  int R;               // query blocks per item (a multiple of 16)
  int chunks;          // items per head: ceil(NB / R)
  float scale_f;
  long long wait_limit;
};

// dynamic shared memory layout (bytes, from a 1024-aligned base)
template <int D>
struct LogTcSmem {
  static constexpr int kDH = D / 64;
  static __host__ __device__ constexpr int q_bytes(int R) { return 3 * kDH * R * 128; }
  static __host__ __device__ constexpr int ring(int R) { return q_bytes(R); }
  static __host__ __device__ constexpr int stage_bytes() { return 128 * 128; }
  static __host__ __device__ constexpr int bars(int R) { return ring(R) + kLogTcStages * stage_bytes(); }
  static __host__ __device__ constexpr int bytes(int R) { return bars(R) + 256; }
};

enum {
  SB_QFULL = 0,
  SB_QFREE = 1,
  SB_KFULL = 2,
  SB_KEMPTY = SB_KFULL + kLogTcStages,
  SB_ACC = SB_KEMPTY + kLogTcStages,     // the item's logits are complete in TMEM
  SB_TFREE = SB_ACC + 1,                 // the drain warps have read TMEM out
  SB_DRAIN = SB_TFREE + 1,               // every product issued has completed (before TMEM is freed)
  SB_COUNT = SB_DRAIN + 1
};

// Row selection: one warp per query-block row.
constexpr int kSelRowsWarps = 4;
constexpr int kHistStride = 17;          // words per lane of a warp's radix-select histogram rows

struct SelRowsParams {
  MaskTcBuffers wb;
  const float* S;      // [BH][NB][NB] fast pooled logits
  unsigned int* refine_count;   // rows listed for refine_rows_kernel (zeroed before the selection)
  int2* refine;        // [BH * NB] listed rows: (row, float bits of the boundary's fast logit)
  uint32_t* bits;
  int32_t* count;
  int16_t* idx;
  long long BH;
  int NB, NW;
  int nX, nY;          // tile grid
  int sta_radius;      // < 0: none
  double p;            // CDF threshold; >= 1 keeps all
  double scale;        // 1 / sqrt(D)
  float scale_f;
};

// Order-preserving maps of float and double onto unsigned integers.
__device__ __forceinline__ uint32_t ord32(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b >> 31) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ unsigned long long ord64(double x) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  return (b >> 63) ? ~b : (b | (1ull << 63));
}
// Selection key: class (2 bits) | order value (46 bits) | 0xFFFF - j.  Larger = earlier in the order.
__device__ __forceinline__ unsigned long long sel_key(unsigned cls, unsigned long long sub46, int j) {
  return (static_cast<unsigned long long>(cls) << 62) | ((sub46 & ((1ull << 46) - 1)) << 16) |
         static_cast<unsigned long long>(0xFFFF - j);
}

// Radix select over 64-bit keys (unique: they carry the block index) with integer masses: the key
// whose cumulative mass in descending key order first reaches `tgt`.  Passes of 4-bit digits,
// starting at the highest bit where the candidates differ.  Each pass builds a 16-bin mass histogram
// of the candidates (the keys that agree with the digits fixed so far): every lane sums its own
// entries into a private row of the warp's shared-memory area `h` (17 words per lane, so the lanes'
// rows fall in different banks), then lane b adds up column b.  The bin where the cumulative mass
// crosses `tgt` fixes the next digit; the select ends once a single candidate is left.  Masses are
// integers and every sum is exact, so the result does not depend on the order of the additions.
// Entries with key 0 are not part of the row.  Per-lane sums must fit 32 bits: NPT masses of at
// most 2^26.
template <int NPT>
__device__ __forceinline__ unsigned long long radix_select(const unsigned long long (&key)[NPT],
                                                          const uint32_t (&M)[NPT], unsigned long long tgt,
                                                          uint32_t* h) {
  const int lane = threadIdx.x & 31;
  // highest bit where the row's keys differ
  unsigned long long first = 0ull, diff = 0ull;
#pragma unroll
  for (int u = 0; u < NPT; ++u)
    if (first == 0ull && key[u] != 0ull) first = key[u];
  {
    const unsigned own = __ballot_sync(0xffffffffu, first != 0ull);
    if (own == 0u) return 0ull;
    first = __shfl_sync(0xffffffffu, first, __ffs(own) - 1);
  }
#pragma unroll
  for (int u = 0; u < NPT; ++u)
    if (key[u] != 0ull) diff |= key[u] ^ first;
  const unsigned dlo = __reduce_or_sync(0xffffffffu, static_cast<unsigned>(diff));
  const unsigned dhi = __reduce_or_sync(0xffffffffu, static_cast<unsigned>(diff >> 32));
  const unsigned long long alld = (static_cast<unsigned long long>(dhi) << 32) | dlo;
  if (alld == 0ull) return first;        // a single entry
  int hi = 63 - __clzll(static_cast<long long>(alld));
  unsigned long long pmask = ~((2ull << hi) - 1ull);   // bits above hi: equal for every entry
  unsigned long long prefix = first & pmask;
  unsigned long long above = 0ull;
  uint32_t* mine = h + lane * kHistStride;
  for (;; hi -= 4) {
    const int lo = hi >= 3 ? hi - 3 : 0;   // digit bits [lo, hi]
    const unsigned long long dmask = (1ull << (hi - lo + 1)) - 1ull;
#pragma unroll
    for (int b = 0; b < 16; ++b) mine[b] = 0u;
    int ncand = 0;
    unsigned long long last = 0ull;
#pragma unroll
    for (int u = 0; u < NPT; ++u) {
      if (key[u] != 0ull && (key[u] & pmask) == prefix) {
        mine[(key[u] >> lo) & dmask] += M[u];
        ++ncand;
        last = key[u];
      }
    }
    // a single candidate left: it is the answer
    const int total_cand = __reduce_add_sync(0xffffffffu, ncand);
    if (total_cand <= 1) {
      const unsigned own = __ballot_sync(0xffffffffu, ncand > 0);
      return own ? __shfl_sync(0xffffffffu, last, __ffs(own) - 1) : 0ull;
    }
    __syncwarp();
    // lanes 0..15 hold the bins in descending digit order: lane i sums column 15 - i
    unsigned long long v = 0ull;
    if (lane < 16) {
      const int d = 15 - lane;
#pragma unroll 8
      for (int l = 0; l < 32; ++l) v += h[l * kHistStride + d];
    }
    __syncwarp();
    unsigned long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned long long o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    // the mass above the candidates plus the candidates' mass reaches tgt, so some bin crosses
    const unsigned hit = __ballot_sync(0xffffffffu, lane < 16 && above + incl >= tgt);
    if (hit == 0u) return 0ull;           // not reached
    const int b = __ffs(hit) - 1;
    above += __shfl_sync(0xffffffffu, incl - v, b);
    prefix |= static_cast<unsigned long long>(15 - b) << lo;
    pmask |= dmask << lo;
    if (lo == 0) {                        // every bit fixed: the unique key with this value
      unsigned long long k = 0ull;
#pragma unroll
      for (int u = 0; u < NPT; ++u)
        if (key[u] != 0ull && key[u] == prefix) k = key[u];
      const unsigned own = __ballot_sync(0xffffffffu, k != 0ull);
      return own ? __shfl_sync(0xffffffffu, k, __ffs(own) - 1) : 0ull;
    }
  }
}

// The boundary on keys of the form class | order | index where class 2 (above the band) and class 0
// (below it) are ordered only coarsely and class 1 (the band) exactly: the mass of class 2 comes
// first, then the band's members in descending key order.  With at most 32 members they are gathered
// one per lane (through `h`), sorted by a bitonic network of shuffles and prefix-summed; otherwise,
// or if the crossing is not among them, radix_select decides.
template <int NPT>
__device__ __forceinline__ unsigned long long band_select(const unsigned long long (&key)[NPT],
                                                         const uint32_t (&M)[NPT], unsigned long long tgt,
                                                         uint32_t* h) {
  const int lane = threadIdx.x & 31;
  uint32_t above_l = 0u;
  int nm_l = 0;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const unsigned cls = static_cast<unsigned>(key[u] >> 62);
    if (key[u] != 0ull && cls == 2u) above_l += M[u];
    if (key[u] != 0ull && cls == 1u) ++nm_l;
  }
  const unsigned long long above = __reduce_add_sync(0xffffffffu, above_l);
  const int nm = __reduce_add_sync(0xffffffffu, nm_l);
  unsigned hit = 0u;
  unsigned long long k = 0ull;
  if (nm > 0 && nm <= 32) {
    unsigned long long* hk = reinterpret_cast<unsigned long long*>(h);   // 32 keys, then 32 masses
    uint32_t* hm = h + 64;
    int off = 0;
#pragma unroll
    for (int u = 0; u < NPT; ++u) {
      const bool mem = key[u] != 0ull && (key[u] >> 62) == 1ull;
      const unsigned m = __ballot_sync(0xffffffffu, mem);
      if (mem) {
        const int slot = off + __popc(m & ((1u << lane) - 1u));
        hk[slot] = key[u];
        hm[slot] = M[u];
      }
      off += __popc(m);
    }
    __syncwarp();
    k = lane < nm ? hk[lane] : 0ull;
    uint32_t w = lane < nm ? hm[lane] : 0u;
    __syncwarp();
    // bitonic sort of the 32 lanes, descending by key (the empty lanes, key 0, sink to the end)
#pragma unroll
    for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
      for (int jj = kk >> 1; jj > 0; jj >>= 1) {
        const unsigned long long ok = __shfl_xor_sync(0xffffffffu, k, jj);
        const uint32_t ow = __shfl_xor_sync(0xffffffffu, w, jj);
        const bool desc = (lane & kk) == 0;      // direction of this lane's sequence (the last: descending)
        const bool lower = (lane & jj) == 0;
        if (lower == desc ? (ok > k) : (ok < k)) {
          k = ok;
          w = ow;
        }
      }
    }
    uint32_t incl = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    hit = __ballot_sync(0xffffffffu, lane < nm && above + incl >= tgt);
  }
  if (hit == 0u) return radix_select<NPT>(key, M, tgt, h);   // a wide band, or a crossing outside it
  return __shfl_sync(0xffffffffu, k, __ffs(hit) - 1);
}

template <int D>
__global__ void __launch_bounds__(kLogTcThreads, 1)
    pooled_logits_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const LogTcParams prm) {
  using L = LogTcSmem<D>;
  constexpr int DH = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const int R = prm.R, ntiles = prm.ntiles, NB = prm.NB;
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(sm + L::bars(R) + 8 * SB_COUNT);
  volatile uint32_t* s_abort = s_misc + 1;
  auto bar = [&](int slot) -> uint32_t { return sbase + L::bars(R) + 8u * slot; };
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
  const long long items = prm.BH * prm.chunks;
  const int tcols = 2 * ntiles * R;
  const uint32_t tmem_cols = tcols <= 32 ? 32u : tcols <= 64 ? 64u : tcols <= 128 ? 128u : tcols <= 256 ? 256u : 512u;
  if (tid == 0) {
    for (int b = 0; b < SB_COUNT; ++b) mbar_init(bar(b), b == SB_TFREE ? kLogTcDrain : 1u);
    fence_mbar_init();
    s_misc[1] = 0;
  }
  if (warp == 1) {
    tmem_alloc(sbase + L::bars(R) + 8 * SB_COUNT, tmem_cols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      bool live = true;
      int n = 0;                 // items of this CTA so far
      long long gst = 0;         // K stages issued
      int armed[kLogTcStages] = {0, 0, 0};
      int qarmed = 0;
      for (long long it = blockIdx.x; it < items && live; it += gridDim.x, ++n) {
        const long long bh = it / prm.chunks;
        const int i0 = static_cast<int>(it - bh * prm.chunks) * R;
        if (n >= 1) wait_live(bar(SB_QFREE), (n - 1) & 1, live);
        if (!live) break;
        mbar_expect_tx(bar(SB_QFULL), 3 * DH * R * 128);
        for (int pc = 0; pc < 3; ++pc)
          for (int h = 0; h < DH; ++h)
            tma_load_4d(sbase + (pc * DH + h) * R * 128, &tmQ, bar(SB_QFULL), 64 * h, i0, static_cast<int>(bh), pc);
        qarmed = n + 1;
        for (int m = 0; m < ntiles && live; ++m)
          for (int h = 0; h < DH && live; ++h)
            for (int pc = 0; pc < 3; ++pc, ++gst) {
              const int s = static_cast<int>(gst % kLogTcStages);
              if (gst >= kLogTcStages)
                wait_live(bar(SB_KEMPTY + s), static_cast<uint32_t>((gst / kLogTcStages) - 1) & 1u, live);
              if (!live) break;
              mbar_expect_tx(bar(SB_KFULL + s), 128 * 128);
              tma_load_4d(sbase + L::ring(R) + s * L::stage_bytes(), &tmK, bar(SB_KFULL + s), 64 * h, 128 * m,
                          static_cast<int>(bh), 3 + pc);
              armed[s] = static_cast<int>(gst / kLogTcStages) + 1;
            }
      }
      // no copy may still be landing when the CTA exits
      for (int s = 0; s < kLogTcStages; ++s)
        if (armed[s] > 0) mbar_wait(bar(SB_KFULL + s), (armed[s] - 1) & 1);
      if (qarmed > 0) mbar_wait(bar(SB_QFULL), (qarmed - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    const uint32_t idesc = idesc_bf16(128, R, 0, 0);   // A = key tile piece (K-major), B = query rows piece
    bool ok = true;
    int n = 0;
    long long gst = 0;
    auto wait_all = [&](int slot, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait_lim(bar(slot), parity, limit));
    };
    for (long long it = blockIdx.x; it < items && ok; it += gridDim.x, ++n) {
      if (!wait_all(SB_QFULL, n & 1)) { ok = false; break; }
      if (n >= 1 && !wait_all(SB_TFREE, (n - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      for (int m = 0; m < ntiles && ok; ++m)
        for (int h = 0; h < DH && ok; ++h)
          for (int pc = 0; pc < 3; ++pc, ++gst) {
            const int s = static_cast<int>(gst % kLogTcStages);
            if (__any_sync(0xffffffffu, *s_abort != 0) ||
                !wait_all(SB_KFULL + s, static_cast<uint32_t>(gst / kLogTcStages) & 1u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t a0 = smem_desc(sbase + L::ring(R) + s * L::stage_bytes(), 16, 1024);
            // key piece pc+1 meets the query pieces whose order sum is at most 4:
            //   D1: (1, 1);  D2: (1, 2), (1, 3), (2, 1), (2, 2), (3, 1)
            const int nq = pc == 0 ? 3 : pc == 1 ? 2 : 1;
            for (int pq = 0; pq < nq; ++pq) {
              const bool d1 = pc == 0 && pq == 0;
              const uint32_t dcol = static_cast<uint32_t>((d1 ? 0 : ntiles) + m) * static_cast<uint32_t>(R);
              const uint64_t b0 = smem_desc(sbase + (pq * DH + h) * R * 128, 16, 1024);
              // first product into D1: (h 0, pc 0, pq 0); into D2: (h 0, pc 0, pq 1)
              const bool first = h == 0 && pc == 0 && pq <= 1;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_f16_elect(tmem + dcol, a0 + static_cast<uint64_t>(kk * 2), b0 + static_cast<uint64_t>(kk * 2),
                               idesc, (first && kk == 0) ? 0u : 1u);
            }
            umma_commit_elect(bar(SB_KEMPTY + s));
          }
      if (!ok) break;
      umma_commit_elect(bar(SB_ACC));
      umma_commit_elect(bar(SB_QFREE));
    }
    if (!ok && lane == 0) *s_abort = 1;
    // every product issued has completed before TMEM is freed
    umma_commit_elect(bar(SB_DRAIN));
    mbar_wait(bar(SB_DRAIN), 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ drain (4 warps): TMEM -> S
    const int qtr = warp & 3;                  // TMEM lane quarter: key blocks 32 qtr .. +31 of each tile
    const uint32_t lrow = static_cast<uint32_t>(32 * qtr) << 16;
    const float scale_f = prm.scale_f;
    bool live = true;
    int n = 0;
    for (long long it = blockIdx.x; it < items; it += gridDim.x, ++n) {
      const long long bh = it / prm.chunks;
      const int i0 = static_cast<int>(it - bh * prm.chunks) * R;
      wait_live(bar(SB_ACC), n & 1, live);
      tc_fence_after();
      // S[bh][i0 + c][j] = (D1 + D2) * scale for key block j = 128 m + 32 qtr + lane: each store of a
      // warp covers 32 consecutive keys of one row
      for (int m = 0; m < ntiles; ++m) {
        const int j = m * 128 + 32 * qtr + lane;
        for (int c0 = 0; c0 < R; c0 += 8) {
          uint32_t a[8], b[8];
          tmem_ld8(tmem + lrow + static_cast<uint32_t>(m * R + c0), a);
          tmem_ld8(tmem + lrow + static_cast<uint32_t>((ntiles + m) * R + c0), b);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int i = i0 + c0 + c;
            if (i < NB && j < NB)
              prm.S[(bh * NB + i) * static_cast<long long>(NB) + j] =
                  (__uint_as_float(a[c]) + __uint_as_float(b[c])) * scale_f;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(SB_TFREE));
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}


// ---------------------------------------------------------------------------
// Row selection.  select_rows_kernel (one warp per row) finds the CDF boundary of every row by
// bisection on its fast logits; a row whose boundary has other blocks within the error band goes to
// a list that refine_rows_kernel settles with float64 logits.  Both write bits, lists and counts
// through emit_row.
// ---------------------------------------------------------------------------

// Bits, list and count of one row from this lane's keep flags (bit u: block lane + 32u), with the
// sliding-tile neighbourhood added.
template <int NPT>
__device__ __forceinline__ void emit_row(const SelRowsParams& prm, long long row, int i, unsigned long long keepm) {
  const int lane = threadIdx.x & 31;
  const int NB = prm.NB, NW = prm.NW;
  const int qx_ = i % prm.nX, qy_ = (i / prm.nX) % prm.nY, qt_ = i / (prm.nX * prm.nY);
  uint32_t* brow = prm.bits + row * NW;
  int16_t* irow = prm.idx + row * NB;
  int base = 0;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const int j = lane + 32 * u;
    bool keep = false;
    if (j < NB) {
      keep = (keepm >> u) & 1ull;
      if (prm.sta_radius >= 0) {
        const int kx = j % prm.nX, ky = (j / prm.nX) % prm.nY, kt = j / (prm.nX * prm.nY);
        const int dmax = max(abs(kt - qt_), max(abs(ky - qy_), abs(kx - qx_)));
        keep = keep || (dmax <= prm.sta_radius);
      }
    }
    const unsigned w = __ballot_sync(0xffffffffu, keep);
    if (u < NW && lane == 0) brow[u] = w;
    if (keep) irow[base + __popc(w & ((1u << lane) - 1u))] = static_cast<int16_t>(j);
    base += __popc(w);
  }
  if (lane == 0) prm.count[row] = base;
}

// Units of the integer masses: 2^21 per the row's largest for rows of at most 1024 blocks, 2^20 for
// rows of at most 2048, so that a row's total stays below 2^32.
template <int NPT>
__device__ __forceinline__ constexpr float mass_unit() { return NPT > 32 ? 1048576.0f : 2097152.0f; }

// A row's fast logits (-inf past NB), max and min, masses e^(s - max) as integers in mass_unit<NPT>()
// of the row's largest (a row sums to at most 2^31, so every sum is exact in 32 bits and independent
// of its order), and the cumulative mass to reach: p of the total, rounded up.
template <int NPT>
__device__ __forceinline__ void load_row(const SelRowsParams& prm, const float* srow, float (&s)[NPT],
                                         uint32_t (&mass)[NPT], float& mx, float& mn, unsigned long long& target) {
  const int lane = threadIdx.x & 31;
  mx = -INFINITY;
  mn = INFINITY;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const bool v = lane + 32 * u < prm.NB;
    s[u] = v ? __ldg(srow + lane + 32 * u) : -INFINITY;
    mx = fmaxf(mx, s[u]);
    if (v) mn = fminf(mn, s[u]);
  }
  mx = warp_max_f32(mx);
  mn = -warp_max_f32(-mn);
  uint32_t lsum = 0u;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    mass[u] = (s[u] != -INFINITY) ? __float2uint_rn(fast_exp2((s[u] - mx) * 1.4426950408889634f) * mass_unit<NPT>()) : 0u;
    lsum += mass[u];
  }
  const uint32_t total = __reduce_add_sync(0xffffffffu, lsum);
  target = static_cast<unsigned long long>(ceil(prm.p * static_cast<double>(total)));
}

// Bound of the fast logits' error for row `row` (see the file header).
__device__ __forceinline__ float logit_error_bound(const SelRowsParams& prm, long long row, long long bh) {
  return 3.0517578125e-05f * prm.scale_f * prm.wb.norm[row] * __uint_as_float(prm.wb.kmax[bh]) * 1.001f;
}

// A row whose band (the blocks with a fast logit within 4E of the boundary block's) holds several
// blocks, settled inside the selecting warp when the band fits it: the band's blocks are gathered one
// per lane (through `gather`, 64 words of shared memory), their float64 logits are computed from the
// pieces and residuals (one warp-wide dot product each), and the lanes are sorted by exact key with a
// shuffle bitonic network and prefix-summed after the mass of the blocks above the band.  Returns
// false, leaving the row to refine_wide_kernel, when the band is wider than a warp or the crossing
// block's fast logit lies in the outer half of the band (a wider band might then reorder it).
template <int D, int NPT>
__device__ __forceinline__ bool band_in_warp(const SelRowsParams& prm, long long row, long long bh,
                                             const float (&s)[NPT], const uint32_t (&mass)[NPT], float sb, float E,
                                             unsigned long long target, uint32_t* gather, unsigned long long& keepm) {
  const int lane = threadIdx.x & 31;
  const int NB = prm.NB;
  const float W = 4.0f * E;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t above_l = 0u;
  int nm = 0;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const bool valid = s[u] != -INFINITY;
    const bool mem = valid && fabsf(s[u] - sb) <= W;
    if (valid && !mem && s[u] > sb) above_l += mass[u];
    const unsigned bal = __ballot_sync(0xffffffffu, mem);
    const int slot = nm + __popc(bal & lt);
    if (mem && slot < 32) {
      gather[slot] = static_cast<uint32_t>(lane + 32 * u);
      gather[32 + slot] = mass[u];
    }
    nm += __popc(bal);
  }
  if (nm > 32) return false;
  __syncwarp();
  const int jm = lane < nm ? static_cast<int>(gather[lane]) : 0;
  uint32_t w = lane < nm ? gather[32 + lane] : 0u;
  __syncwarp();
  const unsigned long long above = __reduce_add_sync(0xffffffffu, above_l);
  // float64 logits of the band's blocks, one warp-wide dot product each
  const long long plane = prm.BH * NB * static_cast<long long>(D);
  double qx[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    const long long o = row * D + lane * (D / 32) + c;
    qx[c] = static_cast<double>(__bfloat162float(prm.wb.pieces[o])) +
            static_cast<double>(__bfloat162float(prm.wb.pieces[plane + o])) +
            static_cast<double>(__bfloat162float(prm.wb.pieces[2 * plane + o])) + static_cast<double>(prm.wb.resid[o]);
  }
  unsigned long long k = 0ull;
  for (int m = 0; m < nm; ++m) {
    const int jj = __shfl_sync(0xffffffffu, jm, m);
    double part = 0.0;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      const long long o = (bh * NB + jj) * static_cast<long long>(D) + lane * (D / 32) + c;
      const double kx = static_cast<double>(__bfloat162float(prm.wb.pieces[3 * plane + o])) +
                        static_cast<double>(__bfloat162float(prm.wb.pieces[4 * plane + o])) +
                        static_cast<double>(__bfloat162float(prm.wb.pieces[5 * plane + o])) +
                        static_cast<double>(prm.wb.resid[plane + o]);
      part = fma(qx[c], kx, part);
    }
    part = warp_sum_f64(part) * prm.scale;
    if (lane == m) k = sel_key(1u, ord64(part) >> 18, jm);
  }
  const unsigned long long k0 = k;               // lane m: the key of the band's m-th block (gather order)
  // bitonic sort of the lanes, descending by key (the empty lanes, key 0, sink to the end)
#pragma unroll
  for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      const unsigned long long ok = __shfl_xor_sync(0xffffffffu, k, jj);
      const uint32_t ow = __shfl_xor_sync(0xffffffffu, w, jj);
      const bool desc = (lane & kk) == 0;
      const bool lower = (lane & jj) == 0;
      if (lower == desc ? (ok > k) : (ok < k)) {
        k = ok;
        w = ow;
      }
    }
  }
  uint32_t incl = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, lane < nm && above + incl >= target);
  if (hit == 0u) return false;                   // not reached: the band and the blocks above it hold the target
  const unsigned long long thr = __shfl_sync(0xffffffffu, k, __ffs(hit) - 1);
  const int jc = 0xFFFF - static_cast<int>(thr & 0xFFFFull);
  // the crossing block's fast logit (every lane finds it in its own registers, one lane owns it)
  float xc = -INFINITY;
#pragma unroll
  for (int u = 0; u < NPT; ++u)
    if (lane + 32 * u == jc) xc = s[u];
  xc = warp_max_f32(xc);
  if (!(fabsf(xc - sb) <= 0.5f * W)) return false;
  // keep: above the band, or in the band at or before the crossing in the exact order
  keepm = 0ull;
  int base = 0;
#pragma unroll
  for (int u = 0; u < NPT; ++u) {
    const bool valid = s[u] != -INFINITY;
    const bool mem = valid && fabsf(s[u] - sb) <= W;
    const unsigned bal = __ballot_sync(0xffffffffu, mem);
    const unsigned long long km = __shfl_sync(0xffffffffu, k0, (base + __popc(bal & lt)) & 31);
    base += __popc(bal);
    const bool keep = mem ? (km >= thr) : (valid && s[u] > sb);
    keepm |= (keep ? 1ull : 0ull) << u;
  }
  return true;
}

// At least four blocks (16 warps) per SM: the rows are latency-bound, so rows in flight matter (for rows
// of 64 blocks per lane that costs a few spilled registers, and is still 4.5 % faster than 8 warps).
template <int D, int NPT>
__global__ void __launch_bounds__(32 * kSelRowsWarps, 4) select_rows_kernel(const SelRowsParams prm) {
  const int lane = threadIdx.x & 31, wk = threadIdx.x >> 5;
  const long long rows = prm.BH * prm.NB;
  const long long row = static_cast<long long>(blockIdx.x) * kSelRowsWarps + wk;
  if (row >= rows) return;                       // whole warps only
  const int NB = prm.NB;
  const long long bh = row / NB;
  const int i = static_cast<int>(row - bh * NB);
  const float* srow = prm.S + row * NB;
  float s[NPT];
  uint32_t mass[NPT];
  float mx, mn;
  unsigned long long target;
  load_row<NPT>(prm, srow, s, mass, mx, mn, target);
  if (!(prm.p < 1.0)) {                          // p = 1 keeps every block
    emit_row<NPT>(prm, row, i, ~0ull);
    return;
  }
  // mass of the blocks whose fast logit is at least t
  auto mass_from = [&](float t) -> unsigned long long {
    uint32_t acc = 0u;
#pragma unroll
    for (int u = 0; u < NPT; ++u) acc += (s[u] >= t) ? mass[u] : 0u;
    return __reduce_add_sync(0xffffffffu, acc);
  };
  const float E = logit_error_bound(prm, row, bh);
  float sb = mx;                                 // fast logit of the boundary block
  if (mass_from(mx) < target) {
    // bisection on the logit value: mass_from(lo) >= target > mass_from(hi) throughout; the boundary
    // block's fast logit lies in [lo, hi), and once that interval is narrower than E / 2 the band
    // settles the order inside it
    float lo = mn, hi = mx;
    for (int it = 0; it < 64 && hi - lo > 0.5f * E; ++it) {
      const float mid = 0.5f * (lo + hi);
      if (!(mid > lo && mid < hi)) break;
      if (mass_from(mid) >= target) lo = mid;
      else hi = mid;
    }
    float c = -INFINITY;
#pragma unroll
    for (int u = 0; u < NPT; ++u)
      if (s[u] >= lo && s[u] < hi) c = fmaxf(c, s[u]);
    sb = warp_max_f32(c);
  }
  // another block within the error band of the boundary: the order there needs float64 logits
  int inband = 0;
#pragma unroll
  for (int u = 0; u < NPT; ++u) inband += (s[u] != -INFINITY && fabsf(s[u] - sb) <= 4.0f * E) ? 1 : 0;
  if (__reduce_add_sync(0xffffffffu, inband) > 1) {
    if (lane == 0) {
      const unsigned k = atomicAdd(prm.refine_count, 1u);
      prm.refine[k] = make_int2(static_cast<int>(row), __float_as_int(sb));
    }
    return;
  }
  unsigned long long keepm = 0ull;
#pragma unroll
  for (int u = 0; u < NPT; ++u) keepm |= (s[u] >= sb ? 1ull : 0ull) << u;
  emit_row<NPT>(prm, row, i, keepm);
}

// The listed rows whose band fits a warp (band_in_warp); the others are flagged in the list (bit 31
// of the row) for refine_wide_kernel.  Persistent: warps walk the list.
template <int D, int NPT>
__global__ void __launch_bounds__(32 * kSelRowsWarps, 4) refine_rows_kernel(const SelRowsParams prm) {
  __shared__ uint32_t s_gather[kSelRowsWarps][64];
  const int lane = threadIdx.x & 31, wk = threadIdx.x >> 5;
  const int NB = prm.NB;
  const unsigned n = *prm.refine_count;
  for (long long e = static_cast<long long>(blockIdx.x) * kSelRowsWarps + wk; e < n;
       e += static_cast<long long>(gridDim.x) * kSelRowsWarps) {
    const int2 ent = prm.refine[e];
    const long long row = ent.x;
    const float sb = __int_as_float(ent.y);
    const long long bh = row / NB;
    const int i = static_cast<int>(row - bh * NB);
    float s[NPT];
    uint32_t mass[NPT];
    float mx, mn;
    unsigned long long target;
    load_row<NPT>(prm, prm.S + row * NB, s, mass, mx, mn, target);
    unsigned long long km;
    if (band_in_warp<D, NPT>(prm, row, bh, s, mass, sb, logit_error_bound(prm, row, bh), target, s_gather[wk], km))
      emit_row<NPT>(prm, row, i, km);
    else if (lane == 0)
      prm.refine[e].x = ent.x | static_cast<int>(0x80000000u);
  }
}

// The flagged rows of the list: exact order inside a band that is widened until the crossing stays in
// its inner half (see the file header), with radix_select over keys of 64 bits.  Persistent: warps walk
// the list and skip the rows refine_rows_kernel settled.
template <int D, int NPT>
__global__ void __launch_bounds__(32 * kSelRowsWarps) refine_wide_kernel(const SelRowsParams prm) {
  __shared__ __align__(16) uint32_t s_hist[kSelRowsWarps][32 * kHistStride];   // rows of 8-byte multiples
  const int lane = threadIdx.x & 31, wk = threadIdx.x >> 5;
  uint32_t* hist = s_hist[wk];
  const int NB = prm.NB;
  const unsigned n = *prm.refine_count;
  for (long long e = static_cast<long long>(blockIdx.x) * kSelRowsWarps + wk; e < n;
       e += static_cast<long long>(gridDim.x) * kSelRowsWarps) {
    const int2 ent = prm.refine[e];
    if (ent.x >= 0) continue;                    // settled by refine_rows_kernel
    const long long row = ent.x & 0x7FFFFFFF;
    const float sb = __int_as_float(ent.y);
    const long long bh = row / NB;
    const int i = static_cast<int>(row - bh * NB);
    const float* srow = prm.S + row * NB;
    float s[NPT];
    uint32_t mass[NPT];
    float mx, mn;
    unsigned long long target;
    load_row<NPT>(prm, srow, s, mass, mx, mn, target);
    auto sv = [&](int u) -> float { return s[u]; };
    const float E = logit_error_bound(prm, row, bh);
    int jb = -1;                                 // the boundary block: the lowest index with the boundary logit
#pragma unroll
    for (int u = NPT - 1; u >= 0; --u) {
      const unsigned eqm = __ballot_sync(0xffffffffu, s[u] == sb);
      if (eqm) jb = 32 * u + __ffs(eqm) - 1;
    }
    unsigned long long key[NPT];
#pragma unroll
    for (int u = 0; u < NPT; ++u) {
      const int j = lane + 32 * u;
      key[u] = (j < NB) ? sel_key(1u, static_cast<unsigned long long>(ord32(s[u])) << 14, j) : 0ull;
    }
    unsigned long long thr = sel_key(1u, static_cast<unsigned long long>(ord32(sb)) << 14, jb);
    uint32_t exact = 0u;          // bit u: key[u] holds the exact order value
    double qx[D / 32];            // this lane's channels of Qp_i, exact, loaded on first use
    bool have_q = false;
    for (float W = 4.0f * E;; W *= 2.0f) {
      bool any = false;
#pragma unroll
      for (int u = 0; u < NPT; ++u) {
        const int j = lane + 32 * u;
        any |= (j < NB) && j != jb && fabsf(sv(u) - sb) <= W;
      }
      if (!__any_sync(0xffffffffu, any)) break;   // the fast order is exact around the boundary
      if (!have_q) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const long long o = row * D + lane * (D / 32) + c;
          const long long plane = prm.BH * NB * static_cast<long long>(D);
          qx[c] = static_cast<double>(__bfloat162float(prm.wb.pieces[o])) +
                  static_cast<double>(__bfloat162float(prm.wb.pieces[plane + o])) +
                  static_cast<double>(__bfloat162float(prm.wb.pieces[2 * plane + o])) +
                  static_cast<double>(prm.wb.resid[o]);
        }
        have_q = true;
      }
      // exact logits for the band (and the boundary block), warp-cooperatively
#pragma unroll
      for (int u = 0; u < NPT; ++u) {
        const int j = lane + 32 * u;
        const bool need = (j < NB) && !((exact >> u) & 1u) && (j == jb || fabsf(sv(u) - sb) <= W);
        unsigned todo = __ballot_sync(0xffffffffu, need);
        while (todo) {
          const int src = __ffs(todo) - 1;
          todo &= todo - 1u;
          const int jj = src + 32 * u;
          const long long plane = prm.BH * NB * static_cast<long long>(D);
          double part = 0.0;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            const long long o = (bh * NB + jj) * static_cast<long long>(D) + lane * (D / 32) + c;
            const double kx = static_cast<double>(__bfloat162float(prm.wb.pieces[3 * plane + o])) +
                              static_cast<double>(__bfloat162float(prm.wb.pieces[4 * plane + o])) +
                              static_cast<double>(__bfloat162float(prm.wb.pieces[5 * plane + o])) +
                              static_cast<double>(prm.wb.resid[plane + o]);
            part = fma(qx[c], kx, part);
          }
          part = warp_sum_f64(part) * prm.scale;
          if (lane == src) {
            key[u] = sel_key(1u, ord64(part) >> 18, jj);
            exact |= 1u << u;
          }
        }
      }
      // keys: exact inside the band, above or below it elsewhere
#pragma unroll
      for (int u = 0; u < NPT; ++u) {
        const int j = lane + 32 * u;
        if (j >= NB) continue;
        const float x = sv(u);
        const bool in = j == jb || fabsf(x - sb) <= W;
        if (!in) {
          key[u] = sel_key(x > sb ? 2u : 0u, static_cast<unsigned long long>(ord32(x)) << 14, j);
        } else if (!((exact >> u) & 1u)) {
          key[u] = sel_key(1u, 0ull, j);   // not reached: every band member is exact by now
        }
      }
      thr = band_select<NPT>(key, mass, target, hist);
      if (thr == 0ull) break;
      const int j2 = 0xFFFF - static_cast<int>(thr & 0xFFFFull);
      if (fabsf(__ldg(srow + j2) - sb) <= 0.5f * W) break;   // the boundary stayed inside the band
    }
    unsigned long long keepm = 0ull;
#pragma unroll
    for (int u = 0; u < NPT; ++u) keepm |= (key[u] != 0ull && key[u] >= thr ? 1ull : 0ull) << u;
    emit_row<NPT>(prm, row, i, keepm);
  }
}

}  // namespace dbst
