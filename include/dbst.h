/*
 * dbst.h — C ABI of the block-sparse tile attention library (libdbst.so).
 *
 * The library implements, on one NVIDIA B200 (sm_100a), the adaptive
 * block-sparse attention described on the page "NABLA: Neighborhood Adaptive
 * Block-Level Attention" (section "Méthodologie : NABLA"): tokens are
 * reordered into 3-D tiles, tiles are mean-pooled, a pooled attention map is
 * thresholded per row by its cumulative distribution, optionally unioned with
 * a sliding-tile neighbourhood, and exact softmax attention runs over the kept
 * tile pairs only.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensors are device memory owned by the caller, contiguous, row-major.
 *   The library never allocates, frees or retains a pointer.
 * - q, k, v, o are bf16 tensors of shape [B, H, N, D] (N = T*Y*X tokens);
 *   "raster" order means token n = (t*Y + y)*X + x, "tiled" order is the
 *   output of dbst_tile_reorder.
 * - A tile (t x y x x = tt x ty x tx tokens) must hold exactly 64 tokens; it is
 *   both the pooling block and the attention block ("block" below).
 *   NB = N / 64 blocks per (b, h).  D must be 64 or 128.
 * - Every device pointer must be 16-byte aligned.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *   enqueued asynchronously; no entry point synchronises except
 *   dbst_get_error.
 * - Argument errors are detected on the host before any launch and return
 *   DBST_EINVAL; nothing is enqueued in that case.  A failed launch returns
 *   DBST_ECUDA.  Device-side faults that the kernels detect themselves (an
 *   expired bounded wait, an out-of-range list entry) set a device error word
 *   that dbst_get_error reports.
 */
#ifndef DBST_H
#define DBST_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DBST_OK = 0,
  DBST_EINVAL = 1,   /* bad argument; nothing was enqueued                      */
  DBST_ECUDA = 2,    /* a CUDA runtime call or launch failed                     */
  DBST_ETIMEOUT = 3, /* a kernel's bounded wait expired; its outputs are invalid */
  DBST_EBOUNDS = 4,  /* a kernel met an out-of-range index list entry            */
  DBST_ETOOLARGE = 5 /* the problem needs more scratch than the fixed static area */
} dbst_status;

/* Shape of one call.  Token grid T x Y x X, tile tt x ty x tx (product 64). */
typedef struct {
  int B, H, D;
  int T, Y, X;
  int tt, ty, tx;
} dbst_geom;

/* Human-readable name of a status code (static string). */
const char* dbst_status_string(int status);

/*
 * Token reorder ("Fractal Flattening", NABLA page, section "Méthodologie").
 * y[b,h,r,:] = x[b,h,n(r),:] where tiled position
 *   r = ((Tt*nY + Ty)*nX + Tx)*64 + (dt*ty + dy)*tx + dx
 * holds raster token n = (t*Y + y)*X + x with Tt, dt = divmod(t, tt), etc.;
 * nY = Y/ty, nX = X/tx.  Tiles come in raster order of tile coordinates, tokens
 * inside a tile in raster order.  Bit-exact copy.  x and y must not overlap.
 */
dbst_status dbst_tile_reorder(const void* x_bf16, void* y_bf16, const dbst_geom* g, void* stream);

/* Inverse of dbst_tile_reorder: tiled [B,H,N,D] -> raster [B,H,N,D]. */
dbst_status dbst_tile_unreorder(const void* y_bf16, void* x_bf16, const dbst_geom* g, void* stream);

/* Bytes of device scratch that the mask builders (dbst_build_block_mask[_raster],
 * dbst_build_sip_mask[_raster]) need for geometry g. */
size_t dbst_mask_workspace_bytes(const dbst_geom* g);

/*
 * Adaptive block mask (NABLA page, "Construction de Masque Adaptatif" and
 * "Intégration Hybride avec STA").
 *   1. Qp, Kp = mean of each block's 64 tiled tokens (float64, exact).
 *   2. A[i,:] = softmax_j(<Qp_i, Kp_j> / sqrt(D)) per (b, h).  Rows of at most
 *      2048 blocks take the logits from the tensor cores (three bf16 pieces of
 *      each mean) and recompute in float64 every key whose logit lies within
 *      the error bound of the selection boundary's, so the order matches the
 *      float64 one; longer rows use float64 logits throughout.
 *   3. Row i keeps the smallest set of key blocks whose mass reaches p:
 *      blocks sorted by A descending (ties: lower index first), keep the
 *      shortest prefix whose cumulative sum is >= p; p == 1 keeps all.
 *   4. If sta_radius >= 0, also keep every key block whose tile lies within
 *      Chebyshev distance sta_radius of the query block's tile (clipped at
 *      the grid edge, no wrap).
 * Inputs: q_tiled, k_tiled bf16 [B,H,N,D] in tiled order.  p in (0, 1].
 * Outputs (caller-allocated):
 *   mask_bits [B,H,NB,ceil(NB/32)] uint32 — bit (j % 32) of word j/32 of row
 *             (b,h,i) is 1 iff key block j is kept;
 *   kv_count  [B,H,NB] int32 — kept blocks per row (>= 1);
 *   kv_idx    [B,H,NB,NB] int16 — row (b,h,i) lists its kept key blocks in
 *             ascending order in its first kv_count entries; the rest of the
 *             row is left untouched.
 * workspace: device scratch of at least dbst_mask_workspace_bytes(g) bytes,
 * 16-byte aligned; contents on entry are ignored.
 */
dbst_status dbst_build_block_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g,
                                  float p, int sta_radius,
                                  uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Expansion of a caller-supplied block mask into the index lists that
 * dbst_block_sparse_attn consumes ("Expansion", NABLA page).  mask_bits has
 * the layout written by dbst_build_block_mask; rows may be empty.
 */
dbst_status dbst_mask_from_bits(const uint32_t* mask_bits, const dbst_geom* g,
                                int32_t* kv_count, int16_t* kv_idx, void* stream);

/*
 * Block-sparse attention ("Expansion", NABLA page): for each (b,h) and query
 * block i with kept key blocks S_i = kv_idx[b,h,i,0:kv_count[b,h,i]],
 *   o[n,:]  = sum_{m in tokens(S_i)} softmax_m(scale * <q_n, k_m>) v[m,:]
 *   lse[n]  = log(sum_{m in tokens(S_i)} exp(scale * <q_n, k_m>))   (natural log)
 * for every query token n of block i; float32 softmax, bf16 output.  A row
 * with kv_count == 0 produces o = 0 and lse = -inf.  q, k, v, o are tiled
 * [B,H,N,D] bf16; lse is [B,H,N] float32 or NULL.  scale <= 0 selects
 * 1/sqrt(D).  List entries must be in [0, NB); an entry outside makes the
 * kernel skip it and report DBST_EBOUNDS through dbst_get_error.
 */
dbst_status dbst_block_sparse_attn(const void* q, const void* k, const void* v, const dbst_geom* g,
                                   const int32_t* kv_count, const int16_t* kv_idx, float scale,
                                   void* o, float* lse, void* stream);

/* Dense attention over all N keys with the same kernel (every list = 0..NB-1). */
dbst_status dbst_dense_attn(const void* q, const void* k, const void* v, const dbst_geom* g,
                            float scale, void* o, float* lse, void* stream);

/*
 * The same three operations on tensors in the caller's raster token order,
 * with the tile reorder ("Fractal Flattening", NABLA page, section
 * "Méthodologie : NABLA") folded into the kernels' own loads and stores
 * instead of separate dbst_tile_reorder / dbst_tile_unreorder passes.
 *   q, k, v, o : raster [B,H,N,D] bf16, token n = (t*Y + y)*X + x
 *   lse        : raster [B,H,N] float32 or NULL
 * The mask outputs (mask_bits, kv_count, kv_idx) are indexed by tile-ordered
 * block as in the tiled entry points, and the workspace is the same
 * (dbst_mask_workspace_bytes).  Results are bit-identical to the tiled entry
 * points applied to dbst_tile_reorder'ed inputs, followed by
 * dbst_tile_unreorder of o (and the same permutation of lse).  Arguments,
 * ownership and errors as for the tiled entry points; in addition q, k, v
 * and o must each be 16-byte aligned (their row stride D*2 bytes always is).
 */
dbst_status dbst_build_block_mask_raster(const void* q, const void* k, const dbst_geom* g,
                                         float p, int sta_radius,
                                         uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx,
                                         void* workspace, size_t workspace_bytes, void* stream);
dbst_status dbst_block_sparse_attn_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                          const int32_t* kv_count, const int16_t* kv_idx,
                                          const int32_t* pairs, float scale,
                                          void* o, float* lse, void* stream);
dbst_status dbst_dense_attn_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                   float scale, void* o, float* lse, void* stream);

/*
 * Schedule for the attention kernel (no counterpart on the pages: it changes
 * which query blocks share a thread block, never which keys a query sees).
 * The kernel runs two 64-token query blocks at a time over the union of their
 * lists; this pairs each block with one of its six face neighbours on the tile
 * grid so that the unions stay small (greedy on the tiles saved, from the mask
 * rows' overlaps), and pairs the rest in ascending order.
 *   mask_bits : [B,H,NB,ceil(NB/32)] uint32 as written by the mask builders
 *   pairs     : out, [B,H,ceil(NB/2)] int32, entry = qa | qb << 16 with
 *               qb = 0xFFFF for a single block; every block of a head appears
 *               exactly once.  Each head's entries come longest first (by
 *               the pair's tiles, ceil(|union| / 2), descending): the
 *               attention kernel starts the longest pairs first.  4-byte
 *               aligned.
 * Pass `pairs` to dbst_block_sparse_attn_raster (NULL there selects fixed
 * pairs of neighbours one tile step apart).  Any order of a head's entries
 * gives the same results; the attention only schedules by it.  An entry
 * naming a block outside [0, NB) makes the attention skip that entry and
 * report DBST_EBOUNDS.
 */
dbst_status dbst_pair_query_blocks(const uint32_t* mask_bits, const dbst_geom* g, int32_t* pairs, void* stream);

/*
 * Allocation-free variant of dbst_build_block_mask.  The paper has no
 * counterpart: this entry point exists for callers that cannot call
 * cudaMalloc or hand the library a workspace — for example a serving loop or
 * plugin host that owns all device memory, forbids allocation once it is
 * running (cudaMalloc may synchronise the device and fragments the host's own
 * pool) and has no spare buffer to lend.
 *
 * It computes exactly what dbst_build_block_mask computes, with the same
 * arguments minus the workspace.  The scratch it needs lives in a fixed
 * static device array of DBST_NOALLOC_SCRATCH_BYTES (64 MiB) inside the
 * library; every GPU that loads the library holds that array until the
 * process exits.  A geometry whose dbst_mask_workspace_bytes exceeds it is
 * rejected with DBST_ETOOLARGE before anything is enqueued (the tiny, small
 * and B=2/H=16/N=16384 shapes fit; the Wan-like and HunyuanVideo-like shapes
 * do not).  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the array's device address once; make that first call before any stream
 * capture begins.  The address is kept for the life of the process, so a
 * cudaDeviceReset (or any other re-creation of the device's primary context)
 * invalidates it: do not call this entry point after one.  All calls share
 * the one array and it keeps the last call's contents; nothing in it needs to
 * start at zero.  Two calls whose kernels
 * overlap on the GPU (different streams without ordering between them) race
 * on the array and produce undefined masks: order them on one stream.
 */
#define DBST_NOALLOC_SCRATCH_BYTES (64u << 20)
dbst_status dbst_build_block_mask_noalloc(const void* q_tiled, const void* k_tiled, const dbst_geom* g,
                                          float p, int sta_radius,
                                          uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx,
                                          void* stream);

/*
 * Transposed block mask for the backward pass.  Row j of mask_bits_t lists
 * the query blocks whose kept set contains key block j:
 *   bit i of mask_bits_t[b,h,j,:]  ==  bit j of mask_bits[b,h,i,:]
 * and (q_count, q_idx) are its index lists, ascending, in the layout of
 * (kv_count, kv_idx).
 *   mask_bits   : [B,H,NB,ceil(NB/32)] uint32, as written by the mask builders
 *   mask_bits_t : out, same shape; must not be mask_bits
 *   q_count     : out, [B,H,NB] int32
 *   q_idx       : out, [B,H,NB,NB] int16 (entries past q_count unspecified)
 */
dbst_status dbst_transpose_block_mask(const uint32_t* mask_bits, const dbst_geom* g, uint32_t* mask_bits_t,
                                      int32_t* q_count, int16_t* q_idx, void* stream);

/* Bytes of device workspace dbst_block_sparse_attn_backward needs (8 per token row). */
size_t dbst_attn_backward_workspace_bytes(const dbst_geom* g);

/*
 * Backward of dbst_block_sparse_attn over the same kept blocks.  The NABLA
 * page (sections "Contributions Clés" and "Résultats Expérimentaux", items on
 * fine-tuning and pre-training) trains with the same adaptive mask; this is
 * the exact gradient of the forward definition for an upstream gradient d_o
 * of o.  For
 * query block i with kept key tokens S_i, P = softmax(scale * q_i k_S^T):
 *   dP      = d_o_i v_S^T
 *   delta_n = sum_m P[n,m] * dP[n,m]       (per query token n; = d_o[n] . o[n])
 *   dS      = P * (dP - delta)
 *   dq_i    = scale * dS k_S
 *   dk_S   += scale * dS^T q_i,   dv_S += P^T d_o_i        (over all i keeping S)
 * P is recomputed from lse in float32 and delta is summed from that P, so the
 * forward's o is not an input.  dS and P are rounded to bf16 before the
 * products, accumulation is float32, outputs are bf16.  A query block with an
 * empty list gets dq = 0 and contributes nothing; a key block no query keeps
 * gets dk = dv = 0.
 *   q, k, v     : tiled [B,H,N,D] bf16, the forward's inputs
 *   lse         : the forward's [B,H,N] float32 log-sum-exp for the same lists
 *   d_o         : tiled [B,H,N,D] bf16
 *   kv_count, kv_idx : the forward's lists
 *   q_count, q_idx   : their transpose (dbst_transpose_block_mask)
 *   scale       : the forward's scale (<= 0 selects 1/sqrt(D))
 *   dq, dk, dv  : out, tiled [B,H,N,D] bf16; every element is written
 *   workspace   : >= dbst_attn_backward_workspace_bytes(g) bytes, 16-byte aligned
 * Two launches on `stream`.  List entries outside [0, NB) are skipped and
 * reported as DBST_EBOUNDS through dbst_get_error.
 */
dbst_status dbst_block_sparse_attn_backward(const void* q, const void* k, const void* v, const float* lse,
                                            const void* d_o, const dbst_geom* g,
                                            const int32_t* kv_count, const int16_t* kv_idx,
                                            const int32_t* q_count, const int16_t* q_idx, float scale,
                                            void* dq, void* dk, void* dv,
                                            void* workspace, size_t workspace_bytes, void* stream);
/* The same on raster-order q, k, v, lse, d_o, dq, dk, dv (lists still indexed by tile-ordered block). */
dbst_status dbst_block_sparse_attn_backward_raster(const void* q, const void* k, const void* v, const float* lse,
                                                   const void* d_o, const dbst_geom* g,
                                                   const int32_t* kv_count, const int16_t* kv_idx,
                                                   const int32_t* q_count, const int16_t* q_idx, float scale,
                                                   void* dq, void* dk, void* dv,
                                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sampled block mask with inclusion-probability weights: SIP on the page
 * "AB-Attention accélère la génération vidéo jusqu'à 2,23× en sautant 92% de
 * l'attention", section "Les trois techniques".  The scores of query block i
 * are its row of the NABLA pooled map (softmax over key blocks of the pooled
 * logits, computed as in dbst_build_block_mask).  Then
 *   pi_ij  = min(1, c_i a_ij), c_i such that sum_j pi_ij = budget; blocks with
 *            c_i a_ij >= 1 are fixed at 1 and c_i is recomputed over the rest
 *            until none joins them; if budget covers every block with a_ij > 0,
 *            all of those get pi = 1
 *   keep   = uniforms[b,h,i,j] < pi_ij
 *   offsets[b,h,i,j] = log(1 / pi_ij) for kept blocks, 0 elsewhere
 * and the bitmask and lists of the kept blocks as dbst_build_block_mask writes
 * them.  Pass offsets to dbst_block_sparse_attn_offsets.
 *   budget   : expected kept blocks per row, > 0 (float64)
 *   uniforms : [B,H,NB,NB] float64 in [0, 1), the caller's random draws
 *   offsets  : out, [B,H,NB,NB] float32
 *   workspace: dbst_mask_workspace_bytes(g) bytes
 * q_tiled, k_tiled as for dbst_build_block_mask (the _raster form takes raster
 * q, k like dbst_build_block_mask_raster).
 */
dbst_status dbst_build_sip_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g, double budget,
                                const double* uniforms, uint32_t* mask_bits, int32_t* kv_count, int16_t* kv_idx,
                                float* offsets, void* workspace, size_t workspace_bytes, void* stream);
dbst_status dbst_build_sip_mask_raster(const void* q, const void* k, const dbst_geom* g, double budget,
                                       const double* uniforms, uint32_t* mask_bits, int32_t* kv_count,
                                       int16_t* kv_idx, float* offsets, void* workspace, size_t workspace_bytes,
                                       void* stream);

/*
 * Block-sparse attention with a logit offset per (query block, key block), as
 * SIP needs it (AB-Attention page, section "Les trois techniques"): for query
 * block i with kept key blocks S_i and every query token n of block i,
 *   o[n]   = sum_{m in tokens(S_i)} softmax_m(scale <q_n, k_m> + off[i, block(m)]) v[m]
 *   lse[n] = log sum_{m in tokens(S_i)} exp(scale <q_n, k_m> + off[i, block(m)])
 * offsets is [B,H,NB,NB] float32 (natural log; read only at kept blocks) or
 * NULL for none.  Runs the kernel of dbst_block_sparse_attn (query blocks
 * paired one tile step apart) with the offset added to the logits before the
 * row max and the exponent, so it costs what the plain forward costs.  An
 * empty row gives o = 0, lse = -inf.  Other arguments as for
 * dbst_block_sparse_attn (the _raster form: raster q, k, v, o, lse); lse may
 * be NULL.
 */
dbst_status dbst_block_sparse_attn_offsets(const void* q, const void* k, const void* v, const dbst_geom* g,
                                           const int32_t* kv_count, const int16_t* kv_idx, const float* offsets,
                                           float scale, void* o, float* lse, void* stream);
dbst_status dbst_block_sparse_attn_offsets_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                  const int32_t* kv_count, const int16_t* kv_idx,
                                                  const float* offsets, float scale, void* o, float* lse,
                                                  void* stream);
/* The same on the query-block schedule `pairs` written by dbst_pair_query_blocks
 * for this mask's bits (required, 4-byte aligned; any order of a head's
 * entries gives the same results, as for dbst_block_sparse_attn_raster). */
dbst_status dbst_block_sparse_attn_offsets_paired(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                  const int32_t* kv_count, const int16_t* kv_idx,
                                                  const float* offsets, const int32_t* pairs, float scale, void* o,
                                                  float* lse, void* stream);
dbst_status dbst_block_sparse_attn_offsets_paired_raster(const void* q, const void* k, const void* v,
                                                         const dbst_geom* g, const int32_t* kv_count,
                                                         const int16_t* kv_idx, const float* offsets,
                                                         const int32_t* pairs, float scale, void* o, float* lse,
                                                         void* stream);

/*
 * Fine-grained mask with key groups of 4 tokens (AB-Attention page, section
 * "Les trois techniques", third technique).  Scoring and selection follow
 * dbst_build_block_mask with a finer key unit: each 64-token query block and
 * each run of 4 consecutive tile-ordered key tokens (a "group"; 16 per block)
 * is mean-pooled in float64, the pooled logits (scale 1/sqrt(D)) are
 * soft-maxed over all N/4 groups of the row, and the row keeps the smallest
 * descending prefix of groups whose mass reaches p (ties to the lower group;
 * p = 1 keeps all).  No sliding-tile union.  Outputs, per (b, h, query block i):
 *   group_mask[b,h,i,j] : uint16, bit r set if group r of key block j (its
 *                         tokens 4r .. 4r+3) is kept
 *   kv_count, kv_idx    : the key blocks with any kept group, ascending (the
 *                         layout of dbst_build_block_mask)
 * NB must be at most 1024.  workspace: dbst_fine_mask_workspace_bytes(g)
 * (float64 means and the [B,H,NB,N/4] float64 logits).  The _raster form
 * takes raster q, k.
 */
size_t dbst_fine_mask_workspace_bytes(const dbst_geom* g);
dbst_status dbst_build_fine_mask(const void* q_tiled, const void* k_tiled, const dbst_geom* g, float p,
                                 uint16_t* group_mask, int32_t* kv_count, int16_t* kv_idx, void* workspace,
                                 size_t workspace_bytes, void* stream);
dbst_status dbst_build_fine_mask_raster(const void* q, const void* k, const dbst_geom* g, float p,
                                        uint16_t* group_mask, int32_t* kv_count, int16_t* kv_idx, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * Attention over the kept 4-token groups: for query block i, the keys are the
 * tokens of the groups that group_mask[b,h,i,:] keeps in the blocks listed by
 * (kv_count, kv_idx); exact softmax over those tokens, o bf16, lse float32
 * (NULL allowed).  Runs a two-sweep kernel (row statistics, then normalised P
 * times V) over the listed blocks with the other groups' columns masked, so it costs
 * whole blocks; gathering the kept groups into full tiles is not done here.
 * group_mask must be 2-byte aligned and is required.  The _raster form takes
 * raster q, k, v, o, lse.
 */
dbst_status dbst_block_sparse_attn_groups(const void* q, const void* k, const void* v, const dbst_geom* g,
                                          const int32_t* kv_count, const int16_t* kv_idx, const uint16_t* group_mask,
                                          float scale, void* o, float* lse, void* stream);
dbst_status dbst_block_sparse_attn_groups_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                 const int32_t* kv_count, const int16_t* kv_idx,
                                                 const uint16_t* group_mask, float scale, void* o, float* lse,
                                                 void* stream);

/*
 * The same attention with the kept groups gathered, the page's own design:
 * each 64-key tile is assembled from 16 kept 4-token groups of the union of a
 * query-block pair's group masks (loaded by index, 4 rows at a time), so only
 * kept groups are computed.  The group masks alone define the keys (no block
 * lists).  NB must be at most 1024; the _raster form also needs tx divisible by
 * 4 (a group is 4 tokens along x).
 */
dbst_status dbst_block_sparse_attn_gather(const void* q, const void* k, const void* v, const dbst_geom* g,
                                          const uint16_t* group_mask, float scale, void* o, float* lse,
                                          void* stream);
dbst_status dbst_block_sparse_attn_gather_raster(const void* q, const void* k, const void* v, const dbst_geom* g,
                                                 const uint16_t* group_mask, float scale, void* o, float* lse,
                                                 void* stream);

/*
 * SQuad two-pass attention (page "SQuad: Sub-Quadratic Attention Distillation
 * for Efficient Video Generation", section "Methodology: SQuad", item
 * "1. SQuad-Attention Operator").  The N tokens of each (b, h) are read as
 * m = N / w windows of w consecutive tokens (token t: window t / w, offset
 * t % w).  With softmax scale `scale` (<= 0 selects 1/sqrt(D)):
 *   local  : o_L[t] = sum over t2 in window(t)      softmax(scale <q_t, k_t2>) v[t2]
 *   global : o[t]   = sum over t2 with t2 % w = t % w  softmax(scale <q_t, k_t2>) o_L[t2]
 * Both passes are the dense attention kernel (float32 softmax, bf16 output; o_L
 * is rounded to bf16 before it feeds the global pass); the global pass runs on
 * window-transposed copies of q, k and o_L.  Six launches on `stream`.
 *   q, k, v, o : [B,H,N,D] bf16, sequence order as given by the caller
 *   w          : window; w and N / w must be multiples of 64 (the page takes
 *                w = sqrt(N), e.g. N = 16384, w = 128)
 *   workspace  : >= dbst_squad_workspace_bytes(B,H,N,D,w) bytes (4 tensors)
 * Unsupported shapes return DBST_EINVAL (and a workspace size of 0).
 */
size_t dbst_squad_workspace_bytes(int B, int H, int N, int D, int w);
dbst_status dbst_squad_attn(const void* q, const void* k, const void* v, int B, int H, int N, int D, int w,
                            float scale, void* o, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then reports (and clears) the first device-side
 * error any kernel of this library recorded since the last call, or a pending
 * CUDA error.  DBST_OK if there was none.
 */
dbst_status dbst_get_error(void* stream);

/*
 * Diagnostic knob (no counterpart on the pages): the limit, in SM clock
 * cycles, of the waits between the roles inside the attention kernels (forward
 * and backward) launched after this call by this process.  A wait that runs
 * out records DBST_ETIMEOUT, the kernel abandons its work (after waiting, with
 * the default limit of about one second, for the copies and tensor-core
 * products it has already issued) and its outputs are undefined.  cycles <= 0
 * restores the default.  It exists so that tests can make a bounded wait
 * expire without faulting anything; production callers leave it alone.
 */
void dbst_set_wait_limit(long long cycles);

#ifdef __cplusplus
}
#endif

#endif /* DBST_H */
