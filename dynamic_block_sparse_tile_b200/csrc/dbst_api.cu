// C ABI of libdbst.so: argument validation, launch configuration, TMA
// descriptors and the device error word.  Every check runs on the host
// before anything is enqueued.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/dbst.h"
#include "attn_sweep.cuh"
#include "fine.cuh"
#include "attn_pair.cuh"
#include "pairing.cuh"
#include "mask.cuh"
#include "mask_tc.cuh"
#include "ptx.cuh"
#include "reorder.cuh"
#include "sip.cuh"
#include "squad.cuh"

namespace {

constexpr int kMaxNB = 4096;   // selection and list kernels keep one row on chip
constexpr int kFineMaxNB = dbst::kFineMaxGroups / 16;   // 4-token groups: 16384 per row at most

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every entry point.
bool geom_ok(const dbst_geom* g) {
  if (!g) return false;
  if (g->B < 1 || g->H < 1) return false;
  if (g->D != 64 && g->D != 128) return false;
  if (g->T < 1 || g->Y < 1 || g->X < 1 || g->tt < 1 || g->ty < 1 || g->tx < 1) return false;
  if (static_cast<long long>(g->tt) * g->ty * g->tx != 64) return false;
  if (g->T % g->tt || g->Y % g->ty || g->X % g->tx) return false;
  const long long N = static_cast<long long>(g->T) * g->Y * g->X;
  if (N / 64 > kMaxNB) return false;
  const long long rows = N * g->B * g->H;
  if (rows >= (1ll << 31)) return false;   // TMA row coordinates are int32
  return true;
}

long long tokens(const dbst_geom* g) { return static_cast<long long>(g->T) * g->Y * g->X; }
int nblocks(const dbst_geom* g) { return static_cast<int>(tokens(g) / 64); }
long long bh_count(const dbst_geom* g) { return static_cast<long long>(g->B) * g->H; }

// Multiprocessors of the current device (the library may drive several devices from one process).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n < 1)
    n = 148;
  return n;
}

// The opt-in to more than 48 KB of dynamic shared memory is a property of a kernel on one device:
// it is set once per (device, kernel) and remembered.
constexpr int kMaxDevices = 64;
bool smem_opt_in(const void* kernel, int bytes) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  struct Entry { const void* fn; int bytes; };
  static std::mutex mu;
  static std::vector<Entry> done[kMaxDevices];
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : done[dev])
    if (e.fn == kernel && e.bytes >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done[dev].push_back({kernel, bytes});
  return true;
}
template <typename K>
bool smem_opt_in(K* kernel, int bytes) {
  return smem_opt_in(reinterpret_cast<const void*>(kernel), bytes);
}

// Limit of the waits between a kernel's roles, in SM clock cycles (dbst_set_wait_limit); 0 = default.
std::atomic<long long> g_wait_limit{0};
long long wait_limit() {
  const long long v = g_wait_limit.load(std::memory_order_relaxed);
  return v > 0 ? v : dbst::kWaitLimitCycles;
}

dbst::TileGeo tile_geo(const dbst_geom* g) {
  dbst::TileGeo t;
  t.N = static_cast<int>(tokens(g));
  t.X = g->X;
  t.Y = g->Y;
  t.tt = g->tt;
  t.ty = g->ty;
  t.tx = g->tx;
  t.nX = g->X / g->tx;
  t.nY = g->Y / g->ty;
  return t;
}

dbst_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? DBST_OK : DBST_ECUDA;
}

dbst_status permute(const void* src, void* dst, const dbst_geom* g, void* stream, int to_tiled) {
  if (!geom_ok(g) || !src || !dst || !aligned16(src) || !aligned16(dst)) return DBST_EINVAL;
  const long long rows = bh_count(g) * tokens(g);
  const long long bytes = rows * g->D * 2;
  const char* a = static_cast<const char*>(src);
  const char* b = static_cast<const char*>(dst);
  if (a < b + bytes && b < a + bytes) return DBST_EINVAL;   // overlapping buffers
  auto s = static_cast<cudaStream_t>(stream);
  const long long bh = bh_count(g);
  if (bh > 65535) return DBST_EINVAL;
  const int N = static_cast<int>(tokens(g));
  const int cpr = g->D / 8;                                   // 16-byte chunks per token row
  const int rows_per_cta = 256 * dbst::kPermuteUnroll / cpr;  // token rows moved by one CTA
  dim3 grid(static_cast<unsigned>((N + rows_per_cta - 1) / rows_per_cta), static_cast<unsigned>(bh));
  const auto* in = static_cast<const uint4*>(src);
  auto* out = static_cast<uint4*>(dst);
  if (g->D == 128)
    dbst::tile_permute_kernel<4><<<grid, 256, 0, s>>>(in, out, tile_geo(g), to_tiled);
  else
    dbst::tile_permute_kernel<3><<<grid, 256, 0, s>>>(in, out, tile_geo(g), to_tiled);
  return launch_status();
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

struct MaskWorkspace {
  size_t qp, kp, s, total;
};
MaskWorkspace mask_workspace(const dbst_geom* g) {
  const size_t nb = static_cast<size_t>(nblocks(g));
  const size_t bh = static_cast<size_t>(bh_count(g));
  MaskWorkspace w;
  w.qp = 0;
  w.kp = align_up(bh * nb * g->D * sizeof(double));
  w.s = w.kp + align_up(bh * nb * g->D * sizeof(double));
  w.total = w.s + align_up(bh * nb * nb * sizeof(double));
  return w;
}

// Tensor-core mask build (rows of at most kMaskTcMaxNB blocks): pool counters, pieces, residuals, norms.
constexpr int kMaskTcMaxNB = 2048;
struct MaskTcWorkspace {
  size_t kmax, pieces, resid, norm, s, refine, total;
};
MaskTcWorkspace mask_tc_workspace(const dbst_geom* g) {
  const size_t nb = static_cast<size_t>(nblocks(g));
  const size_t bh = static_cast<size_t>(bh_count(g));
  const size_t d = static_cast<size_t>(g->D);
  MaskTcWorkspace w;
  w.kmax = 0;                                             // kmax [BH], then the refine-list length
  w.pieces = align_up((bh + 1) * sizeof(unsigned int));
  w.resid = w.pieces + align_up(6 * bh * nb * d * 2);
  w.norm = w.resid + align_up(2 * bh * nb * d * sizeof(float));
  w.s = w.norm + align_up(2 * bh * nb * sizeof(float));   // fast pooled logits [BH][NB][NB] float32
  w.refine = w.s + align_up(bh * nb * nb * sizeof(float)); // rows for the float64 refinement [BH * NB] int2
  w.total = w.refine + align_up(bh * nb * 8);
  return w;
}
// The workspace of every mask builder: the float64 layout of the SIP mask and of rows longer than
// kMaskTcMaxNB blocks, or the tensor-core layout, whichever is larger.
size_t mask_workspace_total(const dbst_geom* g) {
  const size_t a = mask_workspace(g).total, b = mask_tc_workspace(g).total;
  return a > b ? a : b;
}

// ---- TMA descriptors: a [rows, D] bf16 matrix, 64 x 64 boxes, 128-byte swizzle
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap(CUtensorMap* m, const void* base, long long rows, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The mean pieces of the tensor-core mask build, [6][BH][NB][D] bf16, as a 4-D tensor (innermost
// first); one box is `rows` blocks x 64 channels of one piece of one head; rows past NB read as 0.
bool make_tmap_pieces(CUtensorMap* m, const void* base, long long BH, int NB, int D, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(NB), static_cast<cuuint64_t>(BH), 6};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(NB) * D * 2,
                           static_cast<cuuint64_t>(BH) * NB * D * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Query blocks are paired with their neighbour one tile step along the slowest tile axis
// that has more than one tile (time, else height, else width): neighbouring blocks keep
// largely the same key blocks, so the union a pair walks stays close to each list.
int pair_stride(const dbst_geom* g) {
  const int nT = g->T / g->tt, nY = g->Y / g->ty, nX = g->X / g->tx;
  if (nT > 1) return nY * nX;
  if (nY > 1) return nX;
  return 1;
}

// Raster layout [B*H, T, Y, X, D] bf16 as a 5-D tensor (innermost first); one box is one tile's
// tokens x 64 channels, 8 KB, arriving in shared memory in tile order.
bool make_tmap_raster(CUtensorMap* m, const void* base, const dbst_geom* g) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t D = static_cast<cuuint64_t>(g->D);
  cuuint64_t dims[5] = {D, static_cast<cuuint64_t>(g->X), static_cast<cuuint64_t>(g->Y), static_cast<cuuint64_t>(g->T),
                        static_cast<cuuint64_t>(bh_count(g))};
  cuuint64_t strides[4] = {D * 2, D * 2 * dims[1], D * 2 * dims[1] * dims[2], D * 2 * dims[1] * dims[2] * dims[3]};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(g->tx), static_cast<cuuint32_t>(g->ty),
                       static_cast<cuuint32_t>(g->tt), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Boxes of 4 token rows (one 4-token key group) x 64 channels: a [rows, D] matrix, or the raster
// [B*H, T, Y, X, D] tensor with the 4 tokens along x.
bool make_tmap_group(CUtensorMap* m, const void* base, long long rows, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 4};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_tmap_raster_group(CUtensorMap* m, const void* base, const dbst_geom* g) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t D = static_cast<cuuint64_t>(g->D);
  cuuint64_t dims[5] = {D, static_cast<cuuint64_t>(g->X), static_cast<cuuint64_t>(g->Y), static_cast<cuuint64_t>(g->T),
                        static_cast<cuuint64_t>(bh_count(g))};
  cuuint64_t strides[4] = {D * 2, D * 2 * dims[1], D * 2 * dims[1] * dims[2], D * 2 * dims[1] * dims[2] * dims[3]};
  cuuint32_t box[5] = {64, 4, 1, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool RASTER>
dbst_status launch_pair(const void* q, const void* k, const void* v, const dbst_geom* g, const int32_t* cnt,
                        const int16_t* idx, const int32_t* pairs, float scale, void* o, float* lse, cudaStream_t s,
                        const float* offsets = nullptr) {
  const long long rows = bh_count(g) * tokens(g);
  CUtensorMap tq, tk, tv;
  if (RASTER) {
    if (!make_tmap_raster(&tq, q, g) || !make_tmap_raster(&tk, k, g) || !make_tmap_raster(&tv, v, g)) return DBST_ECUDA;
  } else {
    if (!make_tmap(&tq, q, rows, D) || !make_tmap(&tk, k, rows, D) || !make_tmap(&tv, v, rows, D)) return DBST_ECUDA;
  }
  dbst::PairParams p;
  p.tg = tile_geo(g);
  p.kv_count = cnt;
  p.kv_idx = idx;
  p.offsets = offsets;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.NB = nblocks(g);
  p.N = static_cast<int>(tokens(g));
  p.pairs = pairs;
  p.pair_stride = pair_stride(g);
  p.pairs_per_head = pairs ? (p.NB + 1) / 2 : ((p.NB + 2 * p.pair_stride - 1) / (2 * p.pair_stride)) * p.pair_stride;
  const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.wait_limit = wait_limit();
  const int smem = dbst::PairSmem::kBytes + 1024;
  const long long grid = bh_count(g) * p.pairs_per_head;
  if (grid >= (1ll << 31)) return DBST_EINVAL;
  if (offsets != nullptr) {
    if (!smem_opt_in(dbst::pair_attn_kernel<D, RASTER, true>, smem)) return DBST_ECUDA;
    dbst::pair_attn_kernel<D, RASTER, true><<<static_cast<unsigned>(grid), dbst::kPairThreads, smem, s>>>(tq, tk, tv, p);
  } else {
    if (!smem_opt_in(dbst::pair_attn_kernel<D, RASTER>, smem)) return DBST_ECUDA;
    dbst::pair_attn_kernel<D, RASTER><<<static_cast<unsigned>(grid), dbst::kPairThreads, smem, s>>>(tq, tk, tv, p);
  }
  return launch_status();
}

dbst_status attn_common(const void* q, const void* k, const void* v, const dbst_geom* g, const int32_t* cnt,
                        const int16_t* idx, const int32_t* pairs, float scale, void* o, float* lse, void* stream,
                        bool raster) {
  if (!geom_ok(g) || !q || !k || !v || !o) return DBST_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DBST_EINVAL;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return DBST_EINVAL;
  if (!(std::isfinite(scale))) return DBST_EINVAL;
  auto s = static_cast<cudaStream_t>(stream);
  if (pairs && (reinterpret_cast<uintptr_t>(pairs) & 3u)) return DBST_EINVAL;
  if (raster)
    return g->D == 128 ? launch_pair<128, true>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s)
                       : launch_pair<64, true>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s);
  return g->D == 128 ? launch_pair<128, false>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s)
                     : launch_pair<64, false>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s);
}

size_t bwd_workspace(const dbst_geom* g) { return align_up(static_cast<size_t>(bh_count(g) * tokens(g)) * 8u); }

// Backward: the dq pass over the forward's lists (it also writes each query row's (lse * log2 e,
// delta) to `stats`), then the dk/dv pass over the transposed lists.  Own blocks are paired like
// the forward's query blocks.
template <int D, bool RASTER>
dbst_status launch_bwd(const void* q, const void* k, const void* v, const float* lse, const void* dout,
                       const dbst_geom* g, const int32_t* kv_count, const int16_t* kv_idx, const int32_t* q_count,
                       const int16_t* q_idx, float scale, void* dq, void* dk, void* dv, float2* stats,
                       cudaStream_t s) {
  const long long rows = bh_count(g) * tokens(g);
  CUtensorMap tq, tk, tv, tdo;
  if (RASTER) {
    if (!make_tmap_raster(&tq, q, g) || !make_tmap_raster(&tk, k, g) || !make_tmap_raster(&tv, v, g) ||
        !make_tmap_raster(&tdo, dout, g))
      return DBST_ECUDA;
  } else {
    if (!make_tmap(&tq, q, rows, D) || !make_tmap(&tk, k, rows, D) || !make_tmap(&tv, v, rows, D) ||
        !make_tmap(&tdo, dout, rows, D))
      return DBST_ECUDA;
  }
  dbst::SweepParams p{};
  p.tg = tile_geo(g);
  p.lse = lse;
  p.stats = stats;
  p.NB = nblocks(g);
  p.N = static_cast<int>(tokens(g));
  p.pair_stride = pair_stride(g);
  p.pairs_per_head = ((p.NB + 2 * p.pair_stride - 1) / (2 * p.pair_stride)) * p.pair_stride;
  const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.wait_limit = wait_limit();
  const int smem = dbst::SweepSmem::kBytes + 1024;
  if (!smem_opt_in(dbst::sweep_kernel<D, RASTER, 0>, smem) || !smem_opt_in(dbst::sweep_kernel<D, RASTER, 1>, smem))
    return DBST_ECUDA;
  const long long grid = bh_count(g) * p.pairs_per_head;
  if (grid >= (1ll << 31)) return DBST_EINVAL;
  p.count = kv_count;
  p.idx = kv_idx;
  p.out0 = static_cast<__nv_bfloat16*>(dq);
  p.out1 = nullptr;
  dbst::sweep_kernel<D, RASTER, 0><<<static_cast<unsigned>(grid), dbst::kSweepThreads, smem, s>>>(tq, tdo, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  p.count = q_count;
  p.idx = q_idx;
  p.out0 = static_cast<__nv_bfloat16*>(dv);
  p.out1 = static_cast<__nv_bfloat16*>(dk);
  dbst::sweep_kernel<D, RASTER, 1><<<static_cast<unsigned>(grid), dbst::kSweepThreads, smem, s>>>(tk, tv, tq, tdo, p);
  return launch_status();
}

dbst_status bwd_common(const void* q, const void* k, const void* v, const float* lse, const void* dout,
                       const dbst_geom* g, const int32_t* kv_count, const int16_t* kv_idx, const int32_t* q_count,
                       const int16_t* q_idx, float scale, void* dq, void* dk, void* dv, void* workspace,
                       size_t workspace_bytes, void* stream, bool raster) {
  if (!geom_ok(g) || !q || !k || !v || !lse || !dout || !dq || !dk || !dv || !workspace) return DBST_EINVAL;
  if (!kv_count || !kv_idx || !q_count || !q_idx) return DBST_EINVAL;
  for (const void* ptr : {q, k, v, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv), static_cast<const void*>(workspace),
                          static_cast<const void*>(kv_count), static_cast<const void*>(kv_idx),
                          static_cast<const void*>(q_count), static_cast<const void*>(q_idx)})
    if (!aligned16(ptr)) return DBST_EINVAL;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return DBST_EINVAL;
  if (!std::isfinite(scale)) return DBST_EINVAL;
  if (workspace_bytes < bwd_workspace(g)) return DBST_EINVAL;
  auto s = static_cast<cudaStream_t>(stream);
  auto* stats = static_cast<float2*>(workspace);
  if (raster)
    return g->D == 128 ? launch_bwd<128, true>(q, k, v, lse, dout, g, kv_count, kv_idx, q_count, q_idx, scale, dq, dk, dv, stats, s)
                       : launch_bwd<64, true>(q, k, v, lse, dout, g, kv_count, kv_idx, q_count, q_idx, scale, dq, dk, dv, stats, s);
  return g->D == 128 ? launch_bwd<128, false>(q, k, v, lse, dout, g, kv_count, kv_idx, q_count, q_idx, scale, dq, dk, dv, stats, s)
                     : launch_bwd<64, false>(q, k, v, lse, dout, g, kv_count, kv_idx, q_count, q_idx, scale, dq, dk, dv, stats, s);
}

// SQuad shapes: D in {64, 128}; the window w and the window count m = N / w both multiples of 64
// (each pass's sequence is whole 64-token blocks), at most 4096 blocks per sequence.
bool squad_ok(int B, int H, int N, int D, int w) {
  if (B < 1 || H < 1 || N < 1 || (D != 64 && D != 128)) return false;
  if (w < 64 || w % 64 || N % w) return false;
  const int m = N / w;
  if (m < 64 || m % 64) return false;
  if (w / 64 > kMaxNB || m / 64 > kMaxNB) return false;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows >= (1ll << 31)) return false;
  if (static_cast<long long>(H) * m >= (1ll << 31) || static_cast<long long>(H) * w >= (1ll << 31)) return false;
  return true;
}

size_t squad_tensor_bytes(int B, int H, int N, int D) {
  return align_up(static_cast<size_t>(B) * H * N * D * 2);
}

dbst_status window_transpose(const void* src, void* dst, long long heads, int A, int R, int D, cudaStream_t s) {
  const int cpr_log2 = D == 128 ? 4 : 3;
  const long long total = (heads * A * R) << cpr_log2;
  long long grid = (total + 256 * dbst::kPermuteUnroll - 1) / (256 * dbst::kPermuteUnroll);
  const long long cap = static_cast<long long>(sm_count()) * 16;
  if (grid > cap) grid = cap;
  const auto* in = static_cast<const uint4*>(src);
  auto* out = static_cast<uint4*>(dst);
  if (D == 128)
    dbst::window_transpose_kernel<4><<<static_cast<unsigned>(grid), 256, 0, s>>>(in, out, A, R, total);
  else
    dbst::window_transpose_kernel<3><<<static_cast<unsigned>(grid), 256, 0, s>>>(in, out, A, R, total);
  return cudaGetLastError() == cudaSuccess ? DBST_OK : DBST_ECUDA;
}

// Forward with a logit offset per (query block, key block): the two-sweep kernel, MODE 2.
template <int D, bool RASTER>
dbst_status launch_offset_attn(const void* q, const void* k, const void* v, const dbst_geom* g, const int32_t* cnt,
                               const int16_t* idx, const float* offsets, const uint16_t* gmask, float scale, void* o,
                               float* lse, cudaStream_t s) {
  const long long rows = bh_count(g) * tokens(g);
  CUtensorMap tq, tk, tv;
  if (RASTER) {
    if (!make_tmap_raster(&tq, q, g) || !make_tmap_raster(&tk, k, g) || !make_tmap_raster(&tv, v, g)) return DBST_ECUDA;
  } else {
    if (!make_tmap(&tq, q, rows, D) || !make_tmap(&tk, k, rows, D) || !make_tmap(&tv, v, rows, D)) return DBST_ECUDA;
  }
  dbst::SweepParams p{};
  p.tg = tile_geo(g);
  p.count = cnt;
  p.idx = idx;
  p.offsets = offsets;
  p.gmask = gmask;
  p.lse_out = lse;
  p.out0 = static_cast<__nv_bfloat16*>(o);
  p.NB = nblocks(g);
  p.N = static_cast<int>(tokens(g));
  p.pair_stride = pair_stride(g);
  p.pairs_per_head = ((p.NB + 2 * p.pair_stride - 1) / (2 * p.pair_stride)) * p.pair_stride;
  const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.wait_limit = wait_limit();
  const int smem = dbst::SweepSmem::kBytes + 1024;
  if (!smem_opt_in(dbst::sweep_kernel<D, RASTER, 2>, smem)) return DBST_ECUDA;
  const long long grid = bh_count(g) * p.pairs_per_head;
  if (grid >= (1ll << 31)) return DBST_EINVAL;
  // the second tensor-map argument (X2) is not read in this mode
  dbst::sweep_kernel<D, RASTER, 2><<<static_cast<unsigned>(grid), dbst::kSweepThreads, smem, s>>>(tq, tq, tk, tv, p);
  return launch_status();
}

// Attention over the kept 4-token groups, gathered 16 to a 64-key tile: the sweep kernel, MODE 3.
template <int D, bool RASTER>
dbst_status launch_gather_attn(const void* q, const void* k, const void* v, const dbst_geom* g, const uint16_t* gmask,
                               float scale, void* o, float* lse, cudaStream_t s) {
  const long long rows = bh_count(g) * tokens(g);
  CUtensorMap tq, tk, tv;
  if (RASTER) {
    if (!make_tmap_raster(&tq, q, g) || !make_tmap_raster_group(&tk, k, g) || !make_tmap_raster_group(&tv, v, g))
      return DBST_ECUDA;
  } else {
    if (!make_tmap(&tq, q, rows, D) || !make_tmap_group(&tk, k, rows, D) || !make_tmap_group(&tv, v, rows, D))
      return DBST_ECUDA;
  }
  dbst::SweepParams p{};
  p.tg = tile_geo(g);
  p.gmask = gmask;
  p.lse_out = lse;
  p.out0 = static_cast<__nv_bfloat16*>(o);
  p.NB = nblocks(g);
  p.N = static_cast<int>(tokens(g));
  p.pair_stride = pair_stride(g);
  p.pairs_per_head = ((p.NB + 2 * p.pair_stride - 1) / (2 * p.pair_stride)) * p.pair_stride;
  const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.wait_limit = wait_limit();
  const int smem = dbst::SweepLayout<3>::kBytes + 1024;
  if (!smem_opt_in(dbst::sweep_kernel<D, RASTER, 3>, smem)) return DBST_ECUDA;
  const long long grid = bh_count(g) * p.pairs_per_head;
  if (grid >= (1ll << 31)) return DBST_EINVAL;
  // the second tensor-map argument (X2) is not read in this mode
  dbst::sweep_kernel<D, RASTER, 3><<<static_cast<unsigned>(grid), dbst::kSweepThreads, smem, s>>>(tq, tq, tk, tv, p);
  return launch_status();
}

dbst_status gather_common(const void* q, const void* k, const void* v, const dbst_geom* g, const uint16_t* gmask,
                          float scale, void* o, float* lse, void* stream, bool raster) {
  if (!geom_ok(g) || !q || !k || !v || !o || !gmask) return DBST_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (reinterpret_cast<uintptr_t>(gmask) & 1u))
    return DBST_EINVAL;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return DBST_EINVAL;
  if (!std::isfinite(scale)) return DBST_EINVAL;
  if (nblocks(g) > kFineMaxNB) return DBST_EINVAL;    // group union of a pair: at most 16384 entries
  if (raster && g->tx % 4 != 0) return DBST_EINVAL;   // a group must be 4 tokens along x
  auto s = static_cast<cudaStream_t>(stream);
  if (raster)
    return g->D == 128 ? launch_gather_attn<128, true>(q, k, v, g, gmask, scale, o, lse, s)
                       : launch_gather_attn<64, true>(q, k, v, g, gmask, scale, o, lse, s);
  return g->D == 128 ? launch_gather_attn<128, false>(q, k, v, g, gmask, scale, o, lse, s)
                     : launch_gather_attn<64, false>(q, k, v, g, gmask, scale, o, lse, s);
}

dbst_status offset_attn_common(const void* q, const void* k, const void* v, const dbst_geom* g, const int32_t* cnt,
                               const int16_t* idx, const float* offsets, const uint16_t* gmask, float scale, void* o,
                               float* lse, void* stream, bool raster, const int32_t* pairs = nullptr) {
  if (!geom_ok(g) || !q || !k || !v || !o || !cnt || !idx) return DBST_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(cnt) || !aligned16(idx))
    return DBST_EINVAL;
  if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (offsets && (reinterpret_cast<uintptr_t>(offsets) & 3u)) ||
      (gmask && (reinterpret_cast<uintptr_t>(gmask) & 1u)))
    return DBST_EINVAL;
  if (!std::isfinite(scale)) return DBST_EINVAL;
  if (pairs && (reinterpret_cast<uintptr_t>(pairs) & 3u)) return DBST_EINVAL;
  auto s = static_cast<cudaStream_t>(stream);
  if (gmask == nullptr) {   // offsets only: the forward kernel, with the offsets in its exponent
    if (raster)
      return g->D == 128 ? launch_pair<128, true>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s, offsets)
                         : launch_pair<64, true>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s, offsets);
    return g->D == 128 ? launch_pair<128, false>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s, offsets)
                       : launch_pair<64, false>(q, k, v, g, cnt, idx, pairs, scale, o, lse, s, offsets);
  }
  if (raster)
    return g->D == 128 ? launch_offset_attn<128, true>(q, k, v, g, cnt, idx, offsets, gmask, scale, o, lse, s)
                       : launch_offset_attn<64, true>(q, k, v, g, cnt, idx, offsets, gmask, scale, o, lse, s);
  return g->D == 128 ? launch_offset_attn<128, false>(q, k, v, g, cnt, idx, offsets, gmask, scale, o, lse, s)
                     : launch_offset_attn<64, false>(q, k, v, g, cnt, idx, offsets, gmask, scale, o, lse, s);
}

template <int NPT>
bool launch_select(const double* S, const dbst::SelectGeo& sg, long long rows, uint32_t* bits, int32_t* cnt,
                   int16_t* idx, cudaStream_t s) {
  const int smem = 256 * NPT * 16;   // sort keys + masses
  if (smem > 48 * 1024 && !smem_opt_in(dbst::select_kernel<NPT>, smem)) return false;
  dbst::select_kernel<NPT><<<static_cast<unsigned>(rows), 256, smem, s>>>(S, sg, bits, cnt, idx);
  return true;
}

// Steps 1-2 of both mask builders: block means of q and k (tile-ordered or, with `raster`,
// raster-ordered), then the float64 pooled logits S[b,h,i,j] = <qp_i, kp_j> / sqrt(D), into the
// workspace.  The caller has validated the arguments (including B*H <= 65535).
dbst_status pool_and_logits(const void* q, const void* k, const dbst_geom* g, const MaskWorkspace& w, char* ws,
                            cudaStream_t s, bool raster) {
  double* qp = reinterpret_cast<double*>(ws + w.qp);
  double* kp = reinterpret_cast<double*>(ws + w.kp);
  double* S = reinterpret_cast<double*>(ws + w.s);
  const int NB = nblocks(g);
  const long long bh = bh_count(g);
  const long long nblk = bh * NB;
  {  // 1. block mean-pool of q and k
    long long grid = (2 * nblk * 32 + 255) / 256;
    const long long cap = static_cast<long long>(sm_count()) * 8;
    if (grid > cap) grid = cap;
    const auto* qa = static_cast<const uint4*>(q);
    const auto* ka = static_cast<const uint4*>(k);
    const unsigned gr = static_cast<unsigned>(grid);
    const dbst::TileGeo tg = tile_geo(g);
    if (g->D == 128) {
      if (raster) dbst::pool_kernel<128, true><<<gr, 256, 0, s>>>(qa, ka, qp, kp, nblk, NB, tg);
      else dbst::pool_kernel<128, false><<<gr, 256, 0, s>>>(qa, ka, qp, kp, nblk, NB, tg);
    } else {
      if (raster) dbst::pool_kernel<64, true><<<gr, 256, 0, s>>>(qa, ka, qp, kp, nblk, NB, tg);
      else dbst::pool_kernel<64, false><<<gr, 256, 0, s>>>(qa, ka, qp, kp, nblk, NB, tg);
    }
    if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  }
  {  // 2. pooled logits (float64)
    const double scale = 1.0 / std::sqrt(static_cast<double>(g->D));
    dim3 grid((NB + 63) / 64, (NB + 63) / 64, static_cast<unsigned>(bh));
    if (g->D == 128)
      dbst::pooled_logits_kernel<128><<<grid, 256, 0, s>>>(qp, kp, S, NB, scale);
    else
      dbst::pooled_logits_kernel<64><<<grid, 256, 0, s>>>(qp, kp, S, NB, scale);
    if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  }
  return DBST_OK;
}

template <int D, int NPT>
bool launch_select_rows(const dbst::SelRowsParams& prm, cudaStream_t s) {
  const long long rows = prm.BH * prm.NB;
  const long long grid = (rows + dbst::kSelRowsWarps - 1) / dbst::kSelRowsWarps;
  dbst::select_rows_kernel<D, NPT><<<static_cast<unsigned>(grid), 32 * dbst::kSelRowsWarps, 0, s>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return false;
  // the listed rows (a small share): persistent warps walk the list; those whose band does not fit a
  // warp (rare) are flagged for the wide-band kernel, which otherwise only scans the list
  long long rgrid = static_cast<long long>(sm_count()) * 4;
  if (rgrid > grid) rgrid = grid;
  dbst::refine_rows_kernel<D, NPT><<<static_cast<unsigned>(rgrid), 32 * dbst::kSelRowsWarps, 0, s>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return false;
  long long wgrid = static_cast<long long>(sm_count()) * 2;
  if (wgrid > grid) wgrid = grid;
  dbst::refine_wide_kernel<D, NPT><<<static_cast<unsigned>(wgrid), 32 * dbst::kSelRowsWarps, 0, s>>>(prm);
  return cudaGetLastError() == cudaSuccess;
}

template <int D>
bool launch_select_rows_npt(const dbst::SelRowsParams& prm, cudaStream_t s) {
  const int NB = prm.NB;
  if (NB <= 32) return launch_select_rows<D, 1>(prm, s);
  if (NB <= 128) return launch_select_rows<D, 4>(prm, s);
  if (NB <= 256) return launch_select_rows<D, 8>(prm, s);
  if (NB <= 512) return launch_select_rows<D, 16>(prm, s);
  if (NB <= 640) return launch_select_rows<D, 20>(prm, s);
  if (NB <= 1024) return launch_select_rows<D, 32>(prm, s);
  return launch_select_rows<D, 64>(prm, s);
}

// Tensor-core mask build (NB <= kMaskTcMaxNB): the pool (HBM-bound), then the selection (persistent:
// tensor cores for the logits, one warp per row for the CDF selection).
dbst_status build_mask_tc(const void* q, const void* k, const dbst_geom* g, float p, int sta_radius,
                          uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx, char* ws, cudaStream_t s,
                          bool raster) {
  const MaskTcWorkspace w = mask_tc_workspace(g);
  const int NB = nblocks(g), D = g->D;
  const long long BH = bh_count(g);
  dbst::MaskTcBuffers wb;
  wb.kmax = reinterpret_cast<unsigned int*>(ws + w.kmax);
  wb.pieces = reinterpret_cast<__nv_bfloat16*>(ws + w.pieces);
  wb.resid = reinterpret_cast<float*>(ws + w.resid);
  wb.norm = reinterpret_cast<float*>(ws + w.norm);
  if (cudaMemsetAsync(ws + w.kmax, 0, (BH + 1) * sizeof(unsigned int), s) != cudaSuccess) return DBST_ECUDA;
  {  // 1. block means as pieces, residuals and norms
    const long long warps = 2 * BH * NB;
    long long grid = (warps * 32 + dbst::kPoolTcThreads - 1) / dbst::kPoolTcThreads;
    const long long cap = static_cast<long long>(sm_count()) * 8;
    if (grid > cap) grid = cap;
    const auto* qa = static_cast<const uint4*>(q);
    const auto* ka = static_cast<const uint4*>(k);
    const unsigned gr = static_cast<unsigned>(grid);
    const dbst::TileGeo tg = tile_geo(g);
    if (D == 128) {
      if (raster) dbst::pool_pieces_kernel<128, true><<<gr, dbst::kPoolTcThreads, 0, s>>>(qa, ka, wb, BH, NB, tg);
      else dbst::pool_pieces_kernel<128, false><<<gr, dbst::kPoolTcThreads, 0, s>>>(qa, ka, wb, BH, NB, tg);
    } else {
      if (raster) dbst::pool_pieces_kernel<64, true><<<gr, dbst::kPoolTcThreads, 0, s>>>(qa, ka, wb, BH, NB, tg);
      else dbst::pool_pieces_kernel<64, false><<<gr, dbst::kPoolTcThreads, 0, s>>>(qa, ka, wb, BH, NB, tg);
    }
    if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  }
  // 2. pooled logits on the tensor cores, into the float32 map S
  float* S = reinterpret_cast<float*>(ws + w.s);
  dbst::LogTcParams lp;
  lp.wb = wb;
  lp.S = S;
  lp.BH = BH;
  lp.NB = NB;
  lp.ntiles = (NB + 127) / 128;
  // rows per item: the two accumulators of every key tile, 2 * ntiles * R columns, fit TMEM's 512
  lp.R = lp.ntiles <= 3 ? 64 : lp.ntiles <= 5 ? 48 : lp.ntiles <= 8 ? 32 : 16;
  lp.chunks = (NB + lp.R - 1) / lp.R;
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
  lp.scale_f = static_cast<float>(scale);
  lp.wait_limit = wait_limit();
  {
    CUtensorMap tq, tk;
    if (!make_tmap_pieces(&tq, wb.pieces, BH, NB, D, lp.R) || !make_tmap_pieces(&tk, wb.pieces, BH, NB, D, 128))
      return DBST_ECUDA;
    const long long items = BH * lp.chunks;
    const unsigned grid = static_cast<unsigned>(items < sm_count() ? items : sm_count());
    const int smem = (D == 128 ? dbst::LogTcSmem<128>::bytes(lp.R) : dbst::LogTcSmem<64>::bytes(lp.R)) + 1024;
    if (D == 128) {
      if (!smem_opt_in(dbst::pooled_logits_tc_kernel<128>, smem)) return DBST_ECUDA;
      dbst::pooled_logits_tc_kernel<128><<<grid, dbst::kLogTcThreads, smem, s>>>(tq, tk, lp);
    } else {
      if (!smem_opt_in(dbst::pooled_logits_tc_kernel<64>, smem)) return DBST_ECUDA;
      dbst::pooled_logits_tc_kernel<64><<<grid, dbst::kLogTcThreads, smem, s>>>(tq, tk, lp);
    }
    if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  }
  // 3. CDF selection, exactness band, sliding-tile union, lists: one warp per row
  dbst::SelRowsParams prm;
  prm.wb = wb;
  prm.S = S;
  prm.refine_count = wb.kmax + BH;
  prm.refine = reinterpret_cast<int2*>(ws + w.refine);
  prm.bits = mask_bits;
  prm.count = kv_count;
  prm.idx = kv_idx;
  prm.BH = BH;
  prm.NB = NB;
  prm.NW = (NB + 31) / 32;
  prm.nX = g->X / g->tx;
  prm.nY = g->Y / g->ty;
  prm.sta_radius = sta_radius;
  prm.p = static_cast<double>(p);
  prm.scale = scale;
  prm.scale_f = static_cast<float>(scale);
  const bool ok = D == 128 ? launch_select_rows_npt<128>(prm, s) : launch_select_rows_npt<64>(prm, s);
  return ok ? launch_status() : DBST_ECUDA;
}

// Mask build over tile-ordered (raster = false) or raster-ordered (raster = true) q and k.
dbst_status build_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g, float p, int sta_radius,
                       uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx, void* workspace,
                       size_t workspace_bytes, void* stream, bool raster) {
  if (!geom_ok(g) || !q_tiled || !k_tiled || !mask_bits || !kv_count || !kv_idx || !workspace) return DBST_EINVAL;
  if (!aligned16(q_tiled) || !aligned16(k_tiled) || !aligned16(mask_bits) || !aligned16(kv_count) ||
      !aligned16(kv_idx) || !aligned16(workspace))
    return DBST_EINVAL;
  if (!(p > 0.0f && p <= 1.0f)) return DBST_EINVAL;   // also rejects NaN
  const MaskWorkspace w = mask_workspace(g);
  if (workspace_bytes < mask_workspace_total(g)) return DBST_EINVAL;
  if (bh_count(g) > 65535) return DBST_EINVAL;        // grid.z of the pooled-logits launch
  auto s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (nblocks(g) <= kMaskTcMaxNB)
    return build_mask_tc(q_tiled, k_tiled, g, p, sta_radius, mask_bits, kv_count, kv_idx, ws, s, raster);
  double* S = reinterpret_cast<double*>(ws + w.s);
  const int NB = nblocks(g);
  const long long nblk = bh_count(g) * NB;
  const dbst_status st = pool_and_logits(q_tiled, k_tiled, g, w, ws, s, raster);
  if (st != DBST_OK) return st;
  {  // 3. softmax + CDF selection + sliding-tile union + lists
    dbst::SelectGeo sg;
    sg.NB = NB;
    sg.NW = (NB + 31) / 32;
    sg.nX = g->X / g->tx;
    sg.nY = g->Y / g->ty;
    sg.sta_radius = sta_radius;
    sg.p = static_cast<double>(p);
    // rows of 2049 .. kMaxNB blocks (shorter ones take the tensor-core path): one CTA per row
    if (!launch_select<16>(S, sg, nblk, mask_bits, kv_count, kv_idx, s)) return DBST_ECUDA;
  }
  return launch_status();
}

// Fine mask (4-token key groups): float64 query-block and key-group means, the float64 logits of
// every (query block, key group), then one CTA per row for the CDF selection over groups.
struct FineWorkspace {
  size_t qp, kp, s, total;
};
FineWorkspace fine_workspace(const dbst_geom* g) {
  const size_t nb = static_cast<size_t>(nblocks(g)), ng = 16 * nb, bh = static_cast<size_t>(bh_count(g));
  FineWorkspace w;
  w.qp = 0;
  w.kp = align_up(bh * nb * g->D * sizeof(double));
  w.s = w.kp + align_up(bh * ng * g->D * sizeof(double));
  w.total = w.s + align_up(bh * nb * ng * sizeof(double));
  return w;
}

dbst_status build_fine_mask(const void* q, const void* k, const dbst_geom* g, float p, uint16_t* gmask,
                            int32_t* kv_count, int16_t* kv_idx, void* workspace, size_t workspace_bytes, void* stream,
                            bool raster) {
  if (!geom_ok(g) || !q || !k || !gmask || !kv_count || !kv_idx || !workspace) return DBST_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(gmask) || !aligned16(kv_count) || !aligned16(kv_idx) ||
      !aligned16(workspace))
    return DBST_EINVAL;
  if (!(p > 0.0f && p <= 1.0f)) return DBST_EINVAL;
  if (nblocks(g) > kFineMaxNB || bh_count(g) > 65535) return DBST_EINVAL;
  const FineWorkspace w = fine_workspace(g);
  if (workspace_bytes < w.total) return DBST_EINVAL;
  auto s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  double* qp = reinterpret_cast<double*>(ws + w.qp);
  double* kp = reinterpret_cast<double*>(ws + w.kp);
  double* S = reinterpret_cast<double*>(ws + w.s);
  const int NB = nblocks(g), NG = 16 * NB;
  const long long bh = bh_count(g);
  const dbst::TileGeo tg = tile_geo(g);
  const long long cap = static_cast<long long>(sm_count()) * 8;
  auto grid_for = [&](long long warps) {
    long long grid = (warps * 32 + 255) / 256;
    return static_cast<unsigned>(grid > cap ? cap : grid);
  };
  const auto* qa = static_cast<const uint4*>(q);
  const auto* ka = static_cast<const uint4*>(k);
  const long long nq = bh * NB, nk = bh * NG;
  if (g->D == 128) {
    if (raster) {
      dbst::group_pool_kernel<128, true, 64><<<grid_for(nq), 256, 0, s>>>(qa, qp, nq, tg);
      dbst::group_pool_kernel<128, true, 4><<<grid_for(nk), 256, 0, s>>>(ka, kp, nk, tg);
    } else {
      dbst::group_pool_kernel<128, false, 64><<<grid_for(nq), 256, 0, s>>>(qa, qp, nq, tg);
      dbst::group_pool_kernel<128, false, 4><<<grid_for(nk), 256, 0, s>>>(ka, kp, nk, tg);
    }
  } else {
    if (raster) {
      dbst::group_pool_kernel<64, true, 64><<<grid_for(nq), 256, 0, s>>>(qa, qp, nq, tg);
      dbst::group_pool_kernel<64, true, 4><<<grid_for(nk), 256, 0, s>>>(ka, kp, nk, tg);
    } else {
      dbst::group_pool_kernel<64, false, 64><<<grid_for(nq), 256, 0, s>>>(qa, qp, nq, tg);
      dbst::group_pool_kernel<64, false, 4><<<grid_for(nk), 256, 0, s>>>(ka, kp, nk, tg);
    }
  }
  if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  const double scale = 1.0 / std::sqrt(static_cast<double>(g->D));
  dim3 lgrid((NG + 63) / 64, (NB + 63) / 64, static_cast<unsigned>(bh));
  if (g->D == 128)
    dbst::fine_logits_kernel<128><<<lgrid, 256, 0, s>>>(qp, kp, S, NB, NG, scale);
  else
    dbst::fine_logits_kernel<64><<<lgrid, 256, 0, s>>>(qp, kp, S, NB, NG, scale);
  if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  dbst::fine_select_kernel<<<static_cast<unsigned>(bh * NB), dbst::kFineThreads, 0, s>>>(
      S, NB, static_cast<double>(p), gmask, kv_count, kv_idx);
  return launch_status();
}

// SIP mask: pooled logits as for the CDF mask, then the sampled selection with offsets.
dbst_status build_sip_mask(const void* q, const void* k, const dbst_geom* g, double budget, const double* uniforms,
                           uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx, float* offsets, void* workspace,
                           size_t workspace_bytes, void* stream, bool raster) {
  if (!geom_ok(g) || !q || !k || !uniforms || !mask_bits || !kv_count || !kv_idx || !offsets || !workspace)
    return DBST_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(uniforms) || !aligned16(mask_bits) || !aligned16(kv_count) ||
      !aligned16(kv_idx) || !aligned16(offsets) || !aligned16(workspace))
    return DBST_EINVAL;
  if (!(budget > 0.0) || !std::isfinite(budget)) return DBST_EINVAL;
  const MaskWorkspace w = mask_workspace(g);
  if (workspace_bytes < mask_workspace_total(g)) return DBST_EINVAL;
  if (bh_count(g) > 65535) return DBST_EINVAL;
  auto s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const dbst_status st = pool_and_logits(q, k, g, w, ws, s, raster);
  if (st != DBST_OK) return st;
  const int NB = nblocks(g);
  const long long rows = bh_count(g) * NB;
  long long grid = (rows + dbst::kSipWarps - 1) / dbst::kSipWarps;
  const long long cap = static_cast<long long>(sm_count()) * 16;
  if (grid > cap) grid = cap;
  const int smem = dbst::kSipWarps * NB * static_cast<int>(sizeof(double));   // each warp's row of a_j
  if (smem > 48 * 1024 && !smem_opt_in(dbst::sip_select_kernel, smem)) return DBST_ECUDA;
  dbst::sip_select_kernel<<<static_cast<unsigned>(grid), 32 * dbst::kSipWarps, smem, s>>>(
      reinterpret_cast<const double*>(ws + w.s), NB, (NB + 31) / 32, rows, budget, uniforms, mask_bits, kv_count,
      kv_idx, offsets);
  return launch_status();
}

}  // namespace

extern "C" {

const char* dbst_status_string(int status) {
  switch (status) {
    case DBST_OK: return "ok";
    case DBST_EINVAL: return "invalid argument";
    case DBST_ECUDA: return "CUDA error";
    case DBST_ETIMEOUT: return "device wait timed out";
    case DBST_EBOUNDS: return "index list entry out of range";
    case DBST_ETOOLARGE: return "problem exceeds the static scratch of the allocation-free entry point";
    default: return "unknown status";
  }
}

dbst_status dbst_tile_reorder(const void* x, void* y, const dbst_geom* g, void* stream) {
  return permute(x, y, g, stream, 1);
}

dbst_status dbst_tile_unreorder(const void* y, void* x, const dbst_geom* g, void* stream) {
  return permute(y, x, g, stream, 0);
}

size_t dbst_mask_workspace_bytes(const dbst_geom* g) {
  if (!geom_ok(g)) return 0;
  return mask_workspace_total(g);
}

dbst_status dbst_build_block_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g, float p,
                                  int sta_radius, uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return build_mask(q_tiled, k_tiled, g, p, sta_radius, mask_bits, kv_count, kv_idx, workspace, workspace_bytes,
                    stream, false);
}

dbst_status dbst_build_block_mask_raster(const void* q, const void* k, const dbst_geom* g, float p, int sta_radius,
                                         uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  return build_mask(q, k, g, p, sta_radius, mask_bits, kv_count, kv_idx, workspace, workspace_bytes, stream, true);
}

dbst_status dbst_mask_from_bits(const uint32_t* bits, const dbst_geom* g, int32_t* kv_count, int16_t* kv_idx,
                                void* stream) {
  if (!geom_ok(g) || !bits || !kv_count || !kv_idx) return DBST_EINVAL;
  if (!aligned16(bits) || !aligned16(kv_count) || !aligned16(kv_idx)) return DBST_EINVAL;
  const int NB = nblocks(g);
  const long long rows = bh_count(g) * NB;
  long long grid = (rows * 32 + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  if (grid > cap) grid = cap;
  dbst::bits_to_lists_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      bits, NB, (NB + 31) / 32, rows, kv_count, kv_idx);
  return launch_status();
}

dbst_status dbst_block_sparse_attn(const void* q, const void* k, const void* v, const dbst_geom* g,
                                   const int32_t* kv_count, const int16_t* kv_idx, float scale, void* o, float* lse,
                                   void* stream) {
  if (!kv_count || !kv_idx) return DBST_EINVAL;
  if (!aligned16(kv_count) || !aligned16(kv_idx)) return DBST_EINVAL;
  return attn_common(q, k, v, g, kv_count, kv_idx, nullptr, scale, o, lse, stream, false);
}

dbst_status dbst_dense_attn(const void* q, const void* k, const void* v, const dbst_geom* g, float scale, void* o,
                            float* lse, void* stream) {
  return attn_common(q, k, v, g, nullptr, nullptr, nullptr, scale, o, lse, stream, false);
}

dbst_status dbst_block_sparse_attn_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                          const int32_t* kv_count, const int16_t* kv_idx, const int32_t* pairs,
                                          float scale, void* o, float* lse, void* stream) {
  if (!kv_count || !kv_idx) return DBST_EINVAL;
  if (!aligned16(kv_count) || !aligned16(kv_idx)) return DBST_EINVAL;
  return attn_common(q, k, v, g, kv_count, kv_idx, pairs, scale, o, lse, stream, true);
}

dbst_status dbst_dense_attn_raster(const void* q, const void* k, const void* v, const dbst_geom* g, float scale,
                                   void* o, float* lse, void* stream) {
  return attn_common(q, k, v, g, nullptr, nullptr, nullptr, scale, o, lse, stream, true);
}

dbst_status dbst_pair_query_blocks(const uint32_t* mask_bits, const dbst_geom* g, int32_t* pairs, void* stream) {
  if (!geom_ok(g) || !mask_bits || !pairs) return DBST_EINVAL;
  if (!aligned16(mask_bits) || (reinterpret_cast<uintptr_t>(pairs) & 3u)) return DBST_EINVAL;
  const long long bh = bh_count(g);
  if (bh >= (1ll << 31)) return DBST_EINVAL;
  dbst::PairingGeo pg;
  pg.NB = nblocks(g);
  pg.NW = (pg.NB + 31) / 32;
  pg.nX = g->X / g->tx;
  pg.nY = g->Y / g->ty;
  pg.nT = g->T / g->tt;
  const bool stage = dbst::pairing_rows_bytes(pg.NB, pg.NW) <= static_cast<size_t>(dbst::kPairingStageBytes);
  const size_t smem = dbst::pairing_smem_bytes(pg.NB, pg.NW, stage);
  auto kern = stage ? dbst::pair_blocks_kernel<true> : dbst::pair_blocks_kernel<false>;
  if (smem > 48 * 1024 && !smem_opt_in(kern, static_cast<int>(smem))) return DBST_ECUDA;
  kern<<<static_cast<unsigned>(bh), dbst::kPairingThreads, smem, static_cast<cudaStream_t>(stream)>>>(mask_bits, pg,
                                                                                                     pairs);
  return launch_status();
}

dbst_status dbst_transpose_block_mask(const uint32_t* mask_bits, const dbst_geom* g, uint32_t* mask_bits_t,
                                      int32_t* q_count, int16_t* q_idx, void* stream) {
  if (!geom_ok(g) || !mask_bits || !mask_bits_t || !q_count || !q_idx) return DBST_EINVAL;
  if (!aligned16(mask_bits) || !aligned16(mask_bits_t) || !aligned16(q_count) || !aligned16(q_idx))
    return DBST_EINVAL;
  if (mask_bits == mask_bits_t) return DBST_EINVAL;
  const int NB = nblocks(g), NW = (NB + 31) / 32;
  const long long words = bh_count(g) * NB * NW;
  long long grid = (words + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  if (grid > cap) grid = cap;
  auto s = static_cast<cudaStream_t>(stream);
  dbst::transpose_bits_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(mask_bits, mask_bits_t, NB, NW, words);
  if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  return dbst_mask_from_bits(mask_bits_t, g, q_count, q_idx, stream);
}

size_t dbst_attn_backward_workspace_bytes(const dbst_geom* g) {
  if (!geom_ok(g)) return 0;
  return bwd_workspace(g);
}

dbst_status dbst_block_sparse_attn_backward(const void* q, const void* k, const void* v, const float* lse,
                                            const void* d_o, const dbst_geom* g,
                                            const int32_t* kv_count, const int16_t* kv_idx, const int32_t* q_count,
                                            const int16_t* q_idx, float scale, void* dq, void* dk, void* dv,
                                            void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, lse, d_o, g, kv_count, kv_idx, q_count, q_idx, scale, dq, dk, dv, workspace,
                    workspace_bytes, stream, false);
}

dbst_status dbst_block_sparse_attn_backward_raster(const void* q, const void* k, const void* v, const float* lse,
                                                   const void* d_o, const dbst_geom* g,
                                                   const int32_t* kv_count, const int16_t* kv_idx,
                                                   const int32_t* q_count, const int16_t* q_idx, float scale,
                                                   void* dq, void* dk, void* dv, void* workspace,
                                                   size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, lse, d_o, g, kv_count, kv_idx, q_count, q_idx, scale, dq, dk, dv, workspace,
                    workspace_bytes, stream, true);
}

dbst_status dbst_build_sip_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g, double budget,
                                const double* uniforms, uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx,
                                float* offsets, void* workspace, size_t workspace_bytes, void* stream) {
  return build_sip_mask(q_tiled, k_tiled, g, budget, uniforms, mask_bits, kv_count, kv_idx, offsets, workspace,
                        workspace_bytes, stream, false);
}

dbst_status dbst_build_sip_mask_raster(const void* q, const void* k, const dbst_geom* g, double budget,
                                       const double* uniforms, uint32_t* mask_bits, int32_t* kv_count,
                                       int16_t* kv_idx, float* offsets, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  return build_sip_mask(q, k, g, budget, uniforms, mask_bits, kv_count, kv_idx, offsets, workspace,
                        workspace_bytes, stream, true);
}

size_t dbst_fine_mask_workspace_bytes(const dbst_geom* g) {
  if (!geom_ok(g) || nblocks(g) > kFineMaxNB) return 0;
  return fine_workspace(g).total;
}

dbst_status dbst_build_fine_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g, float p,
                                 uint16_t* group_mask, int32_t* kv_count, int16_t* kv_idx, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return build_fine_mask(q_tiled, k_tiled, g, p, group_mask, kv_count, kv_idx, workspace, workspace_bytes, stream,
                         false);
}

dbst_status dbst_build_fine_mask_raster(const void* q, const void* k, const dbst_geom* g, float p,
                                        uint16_t* group_mask, int32_t* kv_count, int16_t* kv_idx, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  return build_fine_mask(q, k, g, p, group_mask, kv_count, kv_idx, workspace, workspace_bytes, stream, true);
}

dbst_status dbst_block_sparse_attn_groups(const void* q, const void* k, const void* v, const dbst_geom* g,
                                          const int32_t* kv_count, const int16_t* kv_idx, const uint16_t* group_mask,
                                          float scale, void* o, float* lse, void* stream) {
  if (!group_mask) return DBST_EINVAL;
  return offset_attn_common(q, k, v, g, kv_count, kv_idx, nullptr, group_mask, scale, o, lse, stream, false);
}

dbst_status dbst_block_sparse_attn_groups_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                 const int32_t* kv_count, const int16_t* kv_idx,
                                                 const uint16_t* group_mask, float scale, void* o, float* lse,
                                                 void* stream) {
  if (!group_mask) return DBST_EINVAL;
  return offset_attn_common(q, k, v, g, kv_count, kv_idx, nullptr, group_mask, scale, o, lse, stream, true);
}

dbst_status dbst_block_sparse_attn_gather(const void* q, const void* k, const void* v, const dbst_geom* g,
                                          const uint16_t* group_mask, float scale, void* o, float* lse,
                                          void* stream) {
  return gather_common(q, k, v, g, group_mask, scale, o, lse, stream, false);
}

dbst_status dbst_block_sparse_attn_gather_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                 const uint16_t* group_mask, float scale, void* o, float* lse,
                                                 void* stream) {
  return gather_common(q, k, v, g, group_mask, scale, o, lse, stream, true);
}

dbst_status dbst_block_sparse_attn_offsets(const void* q, const void* k, const void* v, const dbst_geom* g,
                                           const int32_t* kv_count, const int16_t* kv_idx, const float* offsets,
                                           float scale, void* o, float* lse, void* stream) {
  return offset_attn_common(q, k, v, g, kv_count, kv_idx, offsets, nullptr, scale, o, lse, stream, false);
}

dbst_status dbst_block_sparse_attn_offsets_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                  const int32_t* kv_count, const int16_t* kv_idx,
                                                  const float* offsets, float scale, void* o, float* lse,
                                                  void* stream) {
  return offset_attn_common(q, k, v, g, kv_count, kv_idx, offsets, nullptr, scale, o, lse, stream, true);
}

dbst_status dbst_block_sparse_attn_offsets_paired(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                  const int32_t* kv_count, const int16_t* kv_idx,
                                                  const float* offsets, const int32_t* pairs, float scale, void* o,
                                                  float* lse, void* stream) {
  if (!pairs) return DBST_EINVAL;
  return offset_attn_common(q, k, v, g, kv_count, kv_idx, offsets, nullptr, scale, o, lse, stream, false, pairs);
}

dbst_status dbst_block_sparse_attn_offsets_paired_raster(const void* q, const void* k, const void* v,
                                                         const dbst_geom* g, const int32_t* kv_count,
                                                         const int16_t* kv_idx, const float* offsets,
                                                         const int32_t* pairs, float scale, void* o, float* lse,
                                                         void* stream) {
  if (!pairs) return DBST_EINVAL;
  return offset_attn_common(q, k, v, g, kv_count, kv_idx, offsets, nullptr, scale, o, lse, stream, true, pairs);
}

size_t dbst_squad_workspace_bytes(int B, int H, int N, int D, int w) {
  if (!squad_ok(B, H, N, D, w)) return 0;
  return 4 * squad_tensor_bytes(B, H, N, D);
}

dbst_status dbst_squad_attn(const void* q, const void* k, const void* v, int B, int H, int N, int D, int w,
                            float scale, void* o, void* workspace, size_t workspace_bytes, void* stream) {
  if (!squad_ok(B, H, N, D, w) || !q || !k || !v || !o || !workspace) return DBST_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(workspace)) return DBST_EINVAL;
  if (!std::isfinite(scale)) return DBST_EINVAL;
  const size_t tb = squad_tensor_bytes(B, H, N, D);
  if (workspace_bytes < 4 * tb) return DBST_EINVAL;
  auto s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  void* o_loc = ws;              // local output, later the global output in window-transposed order
  void* qT = ws + tb;
  void* kT = ws + 2 * tb;
  void* o_locT = ws + 3 * tb;
  const int m = N / w;
  const long long heads = static_cast<long long>(B) * H;
  // local pass: every window is a sequence of its own
  const dbst_geom gl = {B, H * m, D, 1, 1, w, 1, 1, 64};
  dbst_status st = attn_common(q, k, v, &gl, nullptr, nullptr, nullptr, scale, o_loc, nullptr, stream, false);
  if (st != DBST_OK) return st;
  // global pass: offset r of every window forms a sequence of m tokens
  if ((st = window_transpose(q, qT, heads, m, w, D, s)) != DBST_OK) return st;
  if ((st = window_transpose(k, kT, heads, m, w, D, s)) != DBST_OK) return st;
  if ((st = window_transpose(o_loc, o_locT, heads, m, w, D, s)) != DBST_OK) return st;
  const dbst_geom gg = {B, H * w, D, 1, 1, m, 1, 1, 64};
  st = attn_common(qT, kT, o_locT, &gg, nullptr, nullptr, nullptr, scale, o_loc, nullptr, stream, false);
  if (st != DBST_OK) return st;
  return window_transpose(o_loc, o, heads, w, m, D, s);
}

void dbst_set_wait_limit(long long cycles) { g_wait_limit.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed); }

dbst_status dbst_get_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DBST_ECUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, dbst::g_error_word, sizeof(word)) != cudaSuccess) return DBST_ECUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(dbst::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return DBST_ECUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return DBST_ECUDA;
  if (word == dbst::kErrTimeout) return DBST_ETIMEOUT;
  if (word == dbst::kErrBounds) return DBST_EBOUNDS;
  return word ? DBST_ECUDA : DBST_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free mask build: the workspace is a fixed static device array.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DBST_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in, so
// the address must come from cudaGetSymbolAddress.
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" dbst_status dbst_build_block_mask_noalloc(const void* q_tiled, const void* k_tiled, const dbst_geom* g,
                                                     float p, int sta_radius, uint32_t* mask_bits,
                                                     int32_t* kv_count, int16_t* kv_idx, void* stream) {
  if (!geom_ok(g)) return DBST_EINVAL;
  if (mask_workspace_total(g) > static_cast<size_t>(DBST_NOALLOC_SCRATCH_BYTES)) return DBST_ETOOLARGE;
  void* scratch = scratch_for_current_device();
  if (scratch == nullptr) return DBST_ECUDA;
  return dbst_build_block_mask(q_tiled, k_tiled, g, p, sta_radius, mask_bits, kv_count, kv_idx, scratch,
                               DBST_NOALLOC_SCRATCH_BYTES, stream);
}
