/*
 * tiered_attn.h -- C ABI of the tiered-precision block-sparse attention library
 * for video diffusion transformers (libtiered_attn.so, sm_100a).
 *
 * The method.  Self-attention over the tokens of a video latent is split into
 * (query-block, key-block) tiles.  A router working from cheap block statistics
 * (pooled block means of Q and K) assigns every tile one of four tiers:
 *   full      computed in bf16;
 *   low       computed in a reduced precision (FP8 e4m3, or NVFP4: e2m1 values
 *             with a ue4m3 scale per 16 elements);
 *   residual  NVFP4 with a second NVFP4 term for x - dequant(x);
 *   skip      replaced by its block means: block j of n_j keys adds
 *             n_j * exp(q . kbar_j * scale) to the softmax denominator and that
 *             weight times vbar_j to the numerator.
 * All tiers are then folded into one flash-style online-softmax pass.
 * Sources: "Triage" (zhuanzhiai paper page, abstract: skip by block means,
 * skim in NVFP4, refine with an NVFP4 residual, router from block statistics,
 * one fused pass); "HierPAS" (conference listing, abstract: progressively
 * reduced precision for less critical regions, cheap pattern estimate);
 * "APT" (Lattice paper summary: two thresholds on attention probability
 * choose selection and precision).  The pooled-mass thresholds below are the
 * tile-level form of those two thresholds.
 *
 * Conventions shared by every entry point.
 *  - Tensors Q, K, V, O are bf16, logically [B, H, N, d], innermost dimension
 *    contiguous; the element strides of the B, H and N dimensions are given in
 *    ta_params.  Base pointers must be 16-byte aligned and stride_n * 2 bytes a
 *    multiple of 16.
 *  - Pointers named *_dev are device pointers; *_host are host pointers (pinned
 *    memory gives asynchronous copies).  The caller owns and allocates every
 *    buffer, including the workspace; no call allocates memory.  State the
 *    library keeps between calls: cached driver entry points, the copy
 *    streams and events of tiered_attn_layer_from_host (created on its first
 *    use on a device), and the fixed device array of
 *    tiered_attn_route_noalloc (part of the module image).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it; only the calls documented as
 *    synchronising wait for the device.
 *  - Every call validates its arguments on the host first and returns a
 *    ta_status without launching anything when they are invalid.  Launch
 *    failures return TA_ERR_CUDA.  Errors found by a kernel (a bounded wait that
 *    ran out) are written to the workspace's status word and read back with
 *    tiered_attn_get_status().
 */
#ifndef TIERED_ATTN_H
#define TIERED_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TA_OK = 0,
  TA_ERR_INVALID_ARG = -1,   /* bad params, null or misaligned pointer        */
  TA_ERR_UNSUPPORTED = -2,   /* valid but not built (e.g. d not in {64,128})  */
  TA_ERR_WORKSPACE = -3,     /* workspace too small                           */
  TA_ERR_CUDA = -4,          /* a CUDA runtime / driver call failed           */
  TA_ERR_TIMEOUT = -5        /* a kernel's bounded wait ran out (device side) */
} ta_status;

typedef enum {
  TA_LOW_NONE = 0,           /* two tiers only: full and skip                 */
  TA_LOW_FP8_E4M3 = 1,       /* low tier in FP8 e4m3, one power-of-two scale per tile */
  TA_LOW_NVFP4 = 2,          /* low tier in NVFP4 (e2m1 + ue4m3 scale per 16)  */
  TA_LOW_NVFP4_RES = 3       /* NVFP4 low tier plus an NVFP4+residual tier    */
} ta_low_format;

/* How tiers are chosen (see tiered_attn_plan). */
typedef enum {
  TA_ROUTER_MASS = 0,        /* cumulative pooled-mass thresholds tau         */
  TA_ROUTER_PRICE = 1,       /* per tile, the tier of least predicted error +
                                price * compute cost ("Triage" abstract)       */
  TA_ROUTER_ENTROPY = 2      /* per query block, keep the ceil(retention *
                                exp(H)) heaviest key blocks, H the entropy of the
                                pooled pattern ("HierPAS" abstract)            */
} ta_router;

/* Tier codes stored in the tier map. */
enum { TA_TIER_SKIP = 0, TA_TIER_LOW = 1, TA_TIER_RES = 2, TA_TIER_FULL = 3 };

typedef struct {
  int32_t B, H, N, d;        /* batch, heads, tokens (N >= 1; the last query and
                                key blocks may be partial, down to one token),
                                head dim (d in {64,128}).  Limits, else
                                TA_ERR_UNSUPPORTED: B * H <= 65535 and
                                ceil(N / block_k) <= 1024 key blocks (the
                                width of the router's per-row sort)            */
  int32_t block_q, block_k;  /* query rows in {64,128}; keys per block in
                                {32,64,128}.  32-key blocks ("FG-Attn",
                                searcharxiv author page, abstract: skipping at
                                M x N sub-tiles) need d = 128, block_q = 128
                                and low NONE, NVFP4 or NVFP4 + residual
                                (else TA_ERR_UNSUPPORTED): the router tiers
                                32-key blocks and the attention kernel packs
                                the kept blocks of one tier four at a time, in
                                list order, into 128-key tiles (one running-
                                max update per tile)                           */
  int32_t low;               /* ta_low_format                                 */
  int32_t n_thresholds;      /* 1 (full only), 2 (full, low), 3 (full, res, low) */
  double  tau[3];            /* ascending cumulative-mass thresholds          */
  int32_t keep_diag_full;    /* 1: key blocks meeting the query block's token
                                range are always full                          */
  int32_t p_offset_log2;     /* o in P' = 2^o exp(s - m): lifts P' into the
                                FP8 / FP4 grids; cancels in O (0..15)          */
  float   softmax_scale;     /* 0 selects 1/sqrt(d)                           */
  int32_t debug_flags;       /* test hooks, 0 in normal use (see TA_DEBUG_*)  */
  int64_t stride_b, stride_h, stride_n;  /* element strides of Q, K, V, O     */
  int32_t router;            /* ta_router                                     */
  double  price;             /* TA_ROUTER_PRICE: error per unit of compute the
                                router pays for a more accurate tier (finite,
                                >= 0); unused by the other routers             */
  double  retention;         /* TA_ROUTER_ENTROPY: kappa, the kept blocks per
                                effective block (finite, > 0); unused otherwise */
  double  tier_cost[4];      /* TA_ROUTER_PRICE: compute cost of a tile in each
                                tier, indexed by tier code (skip, low, res,
                                full), in units of one bf16 tile (finite,
                                >= 0).  All zero selects the costs measured on
                                this library's attention kernel
                                (TA_TIER_COST_* below); unused by the other
                                routers */
} ta_params;

/* Default tier costs of the price router: per-tile time of each tier on this
 * library's fused attention kernel (B200, d = 128, 128 x 128 tiles), relative
 * to a bf16 tile.  A skipped block costs one column of a 128-block skip
 * chunk.  The low tier's cost depends on its format. */
#define TA_TIER_COST_SKIP 0.008
#define TA_TIER_COST_FP8 1.0
#define TA_TIER_COST_NVFP4 1.1
#define TA_TIER_COST_NVFP4_RES 2.2
#define TA_TIER_COST_FULL 1.0

/* Test hook: the attention producer never loads the first K tile, so the
 * kernel's bounded wait runs out and the status word reports TA_ERR_TIMEOUT. */
#define TA_DEBUG_DROP_FIRST_K 1

/* Device pointers into a planned workspace (see tiered_attn_plan_views).
 * BH = B*H, nQb = ceil(N/block_q), nKb = ceil(N/block_k), Np = 32*ceil(N/32).
 * Pointers of data the configured low format does not produce are NULL. */
typedef struct {
  int32_t* status;           /* int32[4]: [0] ta_status of the last kernel error */
  double*  qbar;             /* f64 [BH, nQb, d]  block means of Q            */
  double*  kbar;             /* f64 [BH, nKb, d]  block means of K            */
  uint16_t* kbar_b;          /* bf16 [BH, nKb, d] round-to-nearest-even of kbar */
  uint16_t* vbar_b;          /* bf16 [BH, nKb, d] same for V                  */
  int32_t* n_k;              /* int32 [nKb] keys per key block                */
  double*  logits;           /* f64 [BH, nQb, nKb] pooled logits * scale      */
  double*  mass;             /* f64 [BH, nQb, nKb] pooled block mass M        */
  uint8_t* tier_map;         /* u8  [BH, nQb, nKb] TA_TIER_* per tile          */
  int32_t* row_counts;       /* i32 [BH, nQb, 4] tiles per tier: full, res, low, skip */
  int32_t* row_lists;        /* i32 [BH, nQb, nKb] key blocks by tier: full,
                                then res, low, skip; within a tier by
                                descending pooled mass M, ties by ascending j */
  /* FP8 copies: codes u8 [BH, N, d] (row-major like the input), scales f32
   * per tile [BH, nQb] for Q and [BH, nKb] for K and V.
   * NVFP4 copies: Q, K codes packed two per byte along d, u8 [BH, N, d/2]
   * (element 2c in the low nibble), scales ue4m3 u8 [BH, N, d/16];
   * V codes transposed and packed along tokens, u8 [BH, d, Np/2], scales
   * u8 [BH, Np/16, d] (groups of 16 tokens from token 0; codes and scales of
   * tokens past N are zero, and the pitch Np keeps rows 16-byte aligned). */
  uint8_t* q_codes; uint8_t* k_codes; uint8_t* v_codes;
  void*    q_scales; void* k_scales; void* v_scales;
  /* residual NVFP4 copies (TA_LOW_NVFP4_RES), same layouts as above */
  uint8_t* rq_codes; uint8_t* rk_codes; uint8_t* rv_codes;
  uint8_t* rq_scales; uint8_t* rk_scales; uint8_t* rv_scales;
  /* always NULL: every FP8 and NVFP4 tile runs on the codes and scales, and
   * no bf16 image of a low copy is kept (the fields keep the struct's layout) */
  uint16_t* dq; uint16_t* dk; uint16_t* dv;
  /* always NULL: no bf16 image of the residual copies is kept */
  uint16_t* drq; uint16_t* drk; uint16_t* drv;
  /* TA_ROUTER_PRICE only (NULL otherwise): f64 [BH, nKb, d] the variance of
   * each coordinate over a key block's keys (mean of (k_c - kbar_c)^2), and
   * f64 [BH, nQb, nKb] the skip tier's predicted relative error
   * delta = scale * sqrt(sum_c (qbar_c^2 + qvar_c) kvar_c) */
  double* kvar;
  double* spread;
  /* TA_ROUTER_PRICE only: f64 [BH, nQb, d] the same variances over a query
   * block's queries */
  double* qvar;
} ta_plan_views;

/* Bytes of workspace that tiered_attn_plan / tiered_attn_forward need for
 * `p`; 0 when `p` is invalid or unsupported.  Host only, no device access. */
size_t tiered_attn_workspace_bytes(const ta_params* p);

/* Router + quantiser ("Triage" abstract: the router predicts from block
 * statistics; NVFP4 skim / refine copies).  Reads Q, K, V once: block means of
 * Q, K, V (fp64), the low-precision copies of Q, K, V; then the pooled
 * logits, the
 * n_j-weighted pooled block softmax M, the tiers, and the per-row tile lists.
 * Tiers:
 *  - TA_ROUTER_MASS: by exclusive cumulative mass in (-M, j) order (most
 *    precise tier t with prefix < tau[t], else skip);
 *  - TA_ROUTER_PRICE: each tile's error under tier t is predicted as
 *    M * eps_t, eps the tier's unit roundoff (bf16 2^-8, FP8 2^-4, NVFP4 2^-2,
 *    NVFP4 + residual 2^-4) and, for skip, delta = scale * sqrt(sum_c
 *    (qbar_c^2 + qvar_c) kvar_c) with kvar_c (qvar_c) the variance of
 *    coordinate c over the key (query) block; its cost is the tier's tensor-pipe time relative to an NVFP4 tile
 *    (skip 0, NVFP4 1, FP8 2, NVFP4 + residual 3, bf16 4); the tile takes the
 *    tier of least error + price * cost among those `low` provides (the
 *    cheaper tier on a tie).  tau is then unused but must still be valid;
 *  - TA_ROUTER_ENTROPY: per query block i, H_i = -sum_j M_ij ln M_ij and the
 *    row keeps k_i = min(nKb, max(1, ceil(retention * exp(H_i)))) key blocks,
 *    the first k_i in (-M, j) order, with the precision of the mass rule (the
 *    least precise kept tier where that rule would skip); the rest are skipped.
 * Either way the diagonal blocks are forced full when keep_diag_full, and each
 * row's list holds full, residual, low, then skip blocks, each in (-M, j)
 * order.  Three kernel launches on `stream`.  ws_dev must hold
 * tiered_attn_workspace_bytes(p) bytes, 256-byte aligned; its previous
 * contents are overwritten (the status word is reset).
 * Returns TA_OK when the launches were enqueued. */
ta_status tiered_attn_plan(const ta_params* p, const void* Q_dev, const void* K_dev,
                           const void* V_dev, void* ws_dev, size_t ws_bytes, void* stream);

/* Fused tiered attention over a planned workspace ("Triage" abstract: all
 * tiers in a single pass).  O_dev receives bf16 [B, H, N, d] with the strides of
 * `p`.  Reads the plan in ws_dev and writes only its status word, so one plan
 * serves any number of forwards over the same Q, K, V.  One kernel launch. */
ta_status tiered_attn_forward(const ta_params* p, const void* Q_dev, const void* K_dev,
                              const void* V_dev, void* ws_dev, size_t ws_bytes,
                              void* O_dev, void* stream);

/* Whole layer from host memory: copies Q, K, V (host, [B,H,N,d] with the
 * strides of `p`) into the caller's device buffers, plans, runs the forward and
 * copies O back to O_host.  Host buffers should be pinned for the copies to
 * overlap anything.
 *  - Packed layout (stride_n = d, stride_h = N*d, stride_b = H*N*d) with more
 *    than one (b, h) slice: the layer runs in up to 16 chunks of consecutive
 *    slices (each head is independent, so O is bit for bit that of one plan +
 *    forward).  The copies in of chunk c+1 and out of chunk c-1 overlap the
 *    kernels of chunk c: copies in are enqueued on one library-owned stream,
 *    copies out on another, the kernels on `stream`, ordered by events.  The
 *    copy streams and events are created on first use, once per device, and
 *    kept for the life of the process (no device memory is allocated).  Work
 *    enqueued on `stream` before the call is complete before the first copy
 *    in; `stream` waits for the last copy out.  Calls from several host
 *    threads are serialised while they enqueue.
 *  - Otherwise everything is enqueued on `stream`, one cudaMemcpyAsync per
 *    tensor.
 * Does not synchronise: the caller synchronises `stream` before reading
 * O_host.  Errors as tiered_attn_plan / tiered_attn_forward; TA_ERR_CUDA when a
 * copy, stream or event call fails. */
ta_status tiered_attn_layer_from_host(const ta_params* p, const void* Q_host, const void* K_host,
                                      const void* V_host, void* O_host, void* Q_dev, void* K_dev,
                                      void* V_dev, void* O_dev, void* ws_dev, size_t ws_bytes,
                                      void* stream);

/* Fills `out` with device pointers into ws_dev for workspace layout `p`.  Host
 * only.  TA_ERR_INVALID_ARG for a null argument or invalid `p`. */
ta_status tiered_attn_plan_views(const ta_params* p, void* ws_dev, ta_plan_views* out);

/* Synchronises `stream`, reads the status word of ws_dev and returns it
 * (TA_OK, or the first device-side error such as TA_ERR_TIMEOUT). */
ta_status tiered_attn_get_status(const void* ws_dev, void* stream);

/* The first stage of tiered_attn_plan alone: block means of Q, K, V (and the
 * skip tier's bf16 copies) and the low-precision copies, one kernel launch.
 * The router's output already in ws_dev (tier map, counts, lists) is left as
 * it is, so tiered_attn_prep + tiered_attn_forward runs a layer on a plan made
 * by an earlier tiered_attn_plan: plan reuse across diffusion timesteps ("APT"
 * Lattice paper summary, TAFA: attention probabilities change slowly across
 * timesteps), which skips the pooled logits and the routing.  Same
 * requirements and errors as tiered_attn_plan; `p` must be the plan's. */
ta_status tiered_attn_prep(const ta_params* p, const void* Q_dev, const void* K_dev,
                           const void* V_dev, void* ws_dev, size_t ws_bytes, void* stream);

/* Test entry point: the second stage of tiered_attn_plan alone (pooled
 * logits and routing over the block means already in ws_dev). */
ta_status tiered_attn_route(const ta_params* p, void* ws_dev, size_t ws_bytes, void* stream);

/* Router that allocates nothing (the pages have no counterpart: this is a
 * deployment variant of tiered_attn_plan's routing stage).
 *
 * For callers that cannot allocate device memory: code running inside a host
 * framework that owns all of the GPU's memory (a plugin with a fixed budget),
 * or a latency-critical path where cudaMalloc would synchronise the device.
 * From Q, K, V it writes the tier map (u8 [B*H, nQb, nKb]), the per-row tier
 * counts (i32 [B*H, nQb, 4]) and the per-row lists (i32 [B*H, nQb, nKb]) into
 * caller buffers, exactly as tiered_attn_plan does with the same params (every
 * router: mass, price and entropy); it makes no low-precision copies.  Its
 * intermediate block means, pooled logits and masses (and, for the price
 * router, the block variances and skip spreads) live in one fixed array of
 * TA_ROUTE_NOALLOC_SCRATCH_BYTES in the library's device memory, which every
 * GPU that loads the library holds until the process exits.
 *  - Problems whose intermediates exceed that size (about B*H*nQb*nKb*16 +
 *    B*H*(nQb+nKb)*d*8 + B*H*nKb*d*4 bytes; the price router adds
 *    B*H*nQb*nKb*8 + B*H*(nQb+nKb)*d*8) return TA_ERR_WORKSPACE.
 *  - The first call on a device looks up the array's device address (with that
 *    device current); make that first call before any stream capture.
 *  - All calls share the one array: calls whose work overlaps on the GPU (two
 *    streams, or two threads) race and corrupt each other's results.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Output pointers must be device pointers; Q, K, V 16-byte aligned. */
#define TA_ROUTE_NOALLOC_SCRATCH_BYTES (16u << 20)
ta_status tiered_attn_route_noalloc(const ta_params* p, const void* Q_dev, const void* K_dev,
                                    const void* V_dev, uint8_t* tier_map_dev,
                                    int32_t* row_counts_dev, int32_t* row_lists_dev,
                                    void* stream);

/* Static description of a status code. */
const char* tiered_attn_status_string(ta_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t tiered_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TIERED_ATTN_H */
