// ta_api.cu -- the C ABI of libtiered_attn.so: argument validation, the
// workspace layout, TMA descriptors and the kernel launches.  The library
// allocates no device memory; every buffer, the workspace included, is the
// caller's (tiered_attn_layer_from_host keeps two copy streams and a few
// events per device).
#include <cmath>
#include <cstring>
#include <mutex>

#include "ta_common.cuh"
#include "ta_kernels.cuh"

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kAbsent = ~static_cast<size_t>(0);  // array not in this layout

inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Streams and events of tiered_attn_layer_from_host, created once per device
// on first use and kept for the life of the process.
constexpr int kMaxDevices = 64;
constexpr int kChunks = 16;  // chunks of (b, h) slices a layer is split into
struct CopyStreams {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t ev[2 + 2 * kChunks] = {};
};
CopyStreams g_copy[kMaxDevices];
std::mutex g_copy_mu;

struct Shape {
  int64_t BH, N, d, nQb, nKb, Np;
};

Shape shape_of(const ta_params* p) {
  Shape s;
  s.BH = (int64_t)p->B * p->H;
  s.N = p->N;
  s.d = p->d;
  s.nQb = (p->N + p->block_q - 1) / p->block_q;
  s.nKb = (p->N + p->block_k - 1) / p->block_k;
  // token pitch of the transposed NVFP4 V copy: a multiple of 32 tokens, so that
  // its rows (Np/2 bytes) meet TMA's 16-byte stride rule
  s.Np = 32 * ((p->N + 31) / 32);
  return s;
}

ta_status validate(const ta_params* p) {
  if (!p) return TA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1) return TA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return TA_ERR_UNSUPPORTED;
  if ((p->block_q != 64 && p->block_q != 128) ||
      (p->block_k != 32 && p->block_k != 64 && p->block_k != 128))
    return TA_ERR_UNSUPPORTED;
  // 32-key blocks run packed four to a 128-key tile, in the d = 128 kernel with
  // 128-query blocks, for the bf16 and NVFP4 tiers
  if (p->block_k == 32 && (p->d != 128 || p->block_q != 128 || p->low == TA_LOW_FP8_E4M3))
    return TA_ERR_UNSUPPORTED;
  if (p->low < TA_LOW_NONE || p->low > TA_LOW_NVFP4_RES) return TA_ERR_INVALID_ARG;
  const int want_tau = p->low == TA_LOW_NONE ? 1 : (p->low == TA_LOW_NVFP4_RES ? 3 : 2);
  if (p->n_thresholds != want_tau) return TA_ERR_INVALID_ARG;
  for (int i = 0; i < p->n_thresholds; ++i) {
    if (!std::isfinite(p->tau[i]) || p->tau[i] < 0.0) return TA_ERR_INVALID_ARG;
    if (i > 0 && p->tau[i] < p->tau[i - 1]) return TA_ERR_INVALID_ARG;
  }
  if (p->p_offset_log2 < 0 || p->p_offset_log2 > 15) return TA_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale) || p->softmax_scale < 0.0f) return TA_ERR_INVALID_ARG;
  if (p->keep_diag_full != 0 && p->keep_diag_full != 1) return TA_ERR_INVALID_ARG;
  if (p->router != TA_ROUTER_MASS && p->router != TA_ROUTER_PRICE && p->router != TA_ROUTER_ENTROPY)
    return TA_ERR_INVALID_ARG;
  if (p->router == TA_ROUTER_ENTROPY && !(std::isfinite(p->retention) && p->retention > 0.0))
    return TA_ERR_INVALID_ARG;
  if (p->router == TA_ROUTER_PRICE && !(std::isfinite(p->price) && p->price >= 0.0))
    return TA_ERR_INVALID_ARG;
  if (p->router == TA_ROUTER_PRICE)
    for (int i = 0; i < 4; ++i)
      if (!(std::isfinite(p->tier_cost[i]) && p->tier_cost[i] >= 0.0)) return TA_ERR_INVALID_ARG;
  const Shape s = shape_of(p);
  if (s.nKb > ta::kMaxKeyBlocks) return TA_ERR_UNSUPPORTED;
  if ((int64_t)p->B * p->H > 65535 || s.nQb > 2147483647) return TA_ERR_UNSUPPORTED;
  // TMA: global strides in bytes must be multiples of 16; rows may not overlap.
  if (p->stride_n < p->d || p->stride_h < 1 || p->stride_b < 1) return TA_ERR_INVALID_ARG;
  if ((p->stride_n * 2) % 16 || (p->stride_h * 2) % 16 || (p->stride_b * 2) % 16)
    return TA_ERR_INVALID_ARG;
  return TA_OK;
}


// Workspace layout: byte offsets of every array (kAbsent when not produced).
struct Layout {
  size_t status, n_k, qbar, kbar, kbar_b, vbar_b, logits, mass, tier_map, row_counts, row_lists;
  size_t kvar, spread, qvar;
  size_t q_codes, k_codes, v_codes, q_scales, k_scales, v_scales;
  size_t rq_codes, rk_codes, rv_codes, rq_scales, rk_scales, rv_scales;
  size_t dq, dk, dv, drq, drk, drv;
  size_t total;
};

Layout layout_of(const ta_params* p) {
  const Shape s = shape_of(p);
  Layout L;
  std::memset(&L, 0xFF, sizeof(L));  // every array absent until placed
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  L.status = take(4 * sizeof(int32_t));
  L.n_k = take((size_t)s.nKb * 4);
  L.qbar = take((size_t)s.BH * s.nQb * s.d * 8);
  L.kbar = take((size_t)s.BH * s.nKb * s.d * 8);
  L.kbar_b = take((size_t)s.BH * s.nKb * s.d * 2);
  L.vbar_b = take((size_t)s.BH * s.nKb * s.d * 2);
  L.logits = take((size_t)s.BH * s.nQb * s.nKb * 8);
  L.mass = take((size_t)s.BH * s.nQb * s.nKb * 8);
  L.tier_map = take((size_t)s.BH * s.nQb * s.nKb);
  L.row_counts = take((size_t)s.BH * s.nQb * 4 * 4);
  L.row_lists = take((size_t)s.BH * s.nQb * s.nKb * 4);
  if (p->router == TA_ROUTER_PRICE) {
    L.kvar = take((size_t)s.BH * s.nKb * s.d * 8);
    L.spread = take((size_t)s.BH * s.nQb * s.nKb * 8);
    L.qvar = take((size_t)s.BH * s.nQb * s.d * 8);
  }
  const size_t tok = (size_t)s.BH * s.N * s.d;  // elements of one [BH, N, d] tensor
  if (p->low == TA_LOW_FP8_E4M3) {
    L.q_codes = take(tok);
    L.k_codes = take(tok);
    L.v_codes = take(tok);
    L.q_scales = take((size_t)s.BH * s.nQb * 4);
    L.k_scales = take((size_t)s.BH * s.nKb * 4);
    L.v_scales = take((size_t)s.BH * s.nKb * 4);
  } else if (p->low == TA_LOW_NVFP4 || p->low == TA_LOW_NVFP4_RES) {
    const int reps = p->low == TA_LOW_NVFP4_RES ? 2 : 1;
    for (int r = 0; r < reps; ++r) {
      size_t qc = take(tok / 2), kc = take(tok / 2), vc = take((size_t)s.BH * s.d * s.Np / 2);
      size_t qs = take(tok / 16), ks = take(tok / 16), vs = take((size_t)s.BH * (s.Np / 16) * s.d);
      if (r == 0) {
        L.q_codes = qc; L.k_codes = kc; L.v_codes = vc;
        L.q_scales = qs; L.k_scales = ks; L.v_scales = vs;
      } else {
        L.rq_codes = qc; L.rk_codes = kc; L.rv_codes = vc;
        L.rq_scales = qs; L.rk_scales = ks; L.rv_scales = vs;
      }
    }
  }
  // (no bf16 images of the low copies: FP8 and NVFP4 tiles run on the codes)
  L.total = off;
  return L;
}

template <class T>
T* at(void* ws, size_t off) {
  return off != kAbsent ? reinterpret_cast<T*>(static_cast<char*>(ws) + off) : nullptr;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

ta_status check_ws(const ta_params* p, const void* ws, size_t ws_bytes) {
  if (!ws || !aligned(ws, kAlign)) return TA_ERR_INVALID_ARG;
  if (ws_bytes < layout_of(p).total) return TA_ERR_WORKSPACE;
  return TA_OK;
}

ta_status check_tensor(const void* ptr) {
  return (ptr && aligned(ptr, 16)) ? TA_OK : TA_ERR_INVALID_ARG;
}

}  // namespace

// The price router's tier costs: the caller's, or the measured defaults when
// all four are zero.
void ta_resolve_tier_cost(const ta_params* p, double* cost) {
  bool given = false;
  for (int i = 0; i < 4; ++i) given = given || p->tier_cost[i] != 0.0;
  if (given) {
    for (int i = 0; i < 4; ++i) cost[i] = p->tier_cost[i];
    return;
  }
  cost[TA_TIER_SKIP] = TA_TIER_COST_SKIP;
  cost[TA_TIER_LOW] = p->low == TA_LOW_FP8_E4M3 ? TA_TIER_COST_FP8 : TA_TIER_COST_NVFP4;
  cost[TA_TIER_RES] = TA_TIER_COST_NVFP4_RES;
  cost[TA_TIER_FULL] = TA_TIER_COST_FULL;
}

namespace {

void fill_plan_args(const ta_params* p, const void* Q, const void* K, const void* V, void* ws,
                    ta::PlanArgs& a) {
  const Shape s = shape_of(p);
  const Layout L = layout_of(p);
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.sb = p->stride_b;
  a.sh = p->stride_h;
  a.sn = p->stride_n;
  a.B = p->B;
  a.H = p->H;
  a.N = p->N;
  a.d = p->d;
  a.bq = p->block_q;
  a.bk = p->block_k;
  a.low = p->low;
  a.R = p->block_q > p->block_k ? p->block_q : p->block_k;
  a.nQb = (int)s.nQb;
  a.nKb = (int)s.nKb;
  a.Np = (int)s.Np;
  a.n_tau = p->n_thresholds;
  for (int i = 0; i < 3; ++i) a.tau[i] = i < p->n_thresholds ? p->tau[i] : 0.0;
  a.keep_diag = p->keep_diag_full;
  a.router = p->router;
  a.price = p->price;
  ta_resolve_tier_cost(p, a.cost);
  a.retention = p->retention;
  a.scale = p->softmax_scale > 0.0f ? (double)p->softmax_scale : 1.0 / std::sqrt((double)p->d);
  a.status = at<int>(ws, L.status);
  a.qbar = at<double>(ws, L.qbar);
  a.kbar = at<double>(ws, L.kbar);
  a.kbar_b = at<__nv_bfloat16>(ws, L.kbar_b);
  a.vbar_b = at<__nv_bfloat16>(ws, L.vbar_b);
  a.n_k = at<int>(ws, L.n_k);
  a.logits = at<double>(ws, L.logits);
  a.mass = at<double>(ws, L.mass);
  a.kvar = at<double>(ws, L.kvar);
  a.spread = at<double>(ws, L.spread);
  a.qvar = at<double>(ws, L.qvar);
  a.tier_map = at<uint8_t>(ws, L.tier_map);
  a.row_counts = at<int>(ws, L.row_counts);
  a.row_lists = at<int>(ws, L.row_lists);
  a.q_codes = at<uint8_t>(ws, L.q_codes);
  a.k_codes = at<uint8_t>(ws, L.k_codes);
  a.v_codes = at<uint8_t>(ws, L.v_codes);
  a.q_scales = at<void>(ws, L.q_scales);
  a.k_scales = at<void>(ws, L.k_scales);
  a.v_scales = at<void>(ws, L.v_scales);
  a.rq_codes = at<uint8_t>(ws, L.rq_codes);
  a.rk_codes = at<uint8_t>(ws, L.rk_codes);
  a.rv_codes = at<uint8_t>(ws, L.rv_codes);
  a.rq_scales = at<uint8_t>(ws, L.rq_scales);
  a.rk_scales = at<uint8_t>(ws, L.rk_scales);
  a.rv_scales = at<uint8_t>(ws, L.rv_scales);
}

// ---- TMA descriptors through the driver entry point (no libcuda link) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Byte tensor [BH, rows, inner] (contiguous), box = box_inner bytes x
// box_rows: the packed NVFP4 copies (64-byte boxes, 64-byte swizzle) and the
// FP8 copies (128-byte boxes, 128-byte swizzle).
bool make_map_u8(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int64_t inner,
                 int box_rows, int box_inner) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)inner, (cuuint64_t)(inner * rows)};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            box_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                             : (box_inner == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE),
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map_fp4(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int64_t inner,
                  int box_rows) {
  return make_map_u8(m, base, BH, rows, inner, box_rows, 64);
}

// Transposed NVFP4 V codes [BH, d, Np / 2]: a box is all d rows by the codes of
// one key block.  128-key blocks: 64 bytes, 64-byte swizzle.  32-key blocks:
// 16 bytes, unswizzled, so that the four blocks of a packed tile land as the
// four 16-byte K columns of core matrices of one K-major operand.
bool make_map_vt(CUtensorMap* m, const void* base, int64_t BH, int64_t d, int64_t inner, int block_k) {
  return make_map_u8(m, base, BH, d, inner, (int)d, block_k / 2);
}

// bf16 tensor [B, H, N, d] (element strides sb, sh, sn), box = 64 x rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int B, int H, int N, int d, int64_t sb, int64_t sh,
              int64_t sn, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)sn * 2, (cuuint64_t)sh * 2, (cuuint64_t)sb * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

int32_t tiered_attn_version(void) { return 100; }

const char* tiered_attn_status_string(ta_status s) {
  switch (s) {
    case TA_OK: return "ok";
    case TA_ERR_INVALID_ARG: return "invalid argument";
    case TA_ERR_UNSUPPORTED: return "unsupported configuration";
    case TA_ERR_WORKSPACE: return "workspace too small";
    case TA_ERR_CUDA: return "CUDA error";
    case TA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

size_t tiered_attn_workspace_bytes(const ta_params* p) {
  if (validate(p) != TA_OK) return 0;
  return layout_of(p).total;
}

ta_status tiered_attn_plan_views(const ta_params* p, void* ws, ta_plan_views* out) {
  if (!out || !ws) return TA_ERR_INVALID_ARG;
  const ta_status st = validate(p);
  if (st != TA_OK) return st;
  const Layout L = layout_of(p);
  out->status = at<int32_t>(ws, L.status);
  out->qbar = at<double>(ws, L.qbar);
  out->kbar = at<double>(ws, L.kbar);
  out->kbar_b = at<uint16_t>(ws, L.kbar_b);
  out->vbar_b = at<uint16_t>(ws, L.vbar_b);
  out->n_k = at<int32_t>(ws, L.n_k);
  out->logits = at<double>(ws, L.logits);
  out->mass = at<double>(ws, L.mass);
  out->tier_map = at<uint8_t>(ws, L.tier_map);
  out->row_counts = at<int32_t>(ws, L.row_counts);
  out->row_lists = at<int32_t>(ws, L.row_lists);
  out->q_codes = at<uint8_t>(ws, L.q_codes);
  out->k_codes = at<uint8_t>(ws, L.k_codes);
  out->v_codes = at<uint8_t>(ws, L.v_codes);
  out->q_scales = at<void>(ws, L.q_scales);
  out->k_scales = at<void>(ws, L.k_scales);
  out->v_scales = at<void>(ws, L.v_scales);
  out->rq_codes = at<uint8_t>(ws, L.rq_codes);
  out->rk_codes = at<uint8_t>(ws, L.rk_codes);
  out->rv_codes = at<uint8_t>(ws, L.rv_codes);
  out->rq_scales = at<uint8_t>(ws, L.rq_scales);
  out->rk_scales = at<uint8_t>(ws, L.rk_scales);
  out->rv_scales = at<uint8_t>(ws, L.rv_scales);
  out->dq = at<uint16_t>(ws, L.dq);
  out->dk = at<uint16_t>(ws, L.dk);
  out->dv = at<uint16_t>(ws, L.dv);
  out->drq = at<uint16_t>(ws, L.drq);
  out->drk = at<uint16_t>(ws, L.drk);
  out->drv = at<uint16_t>(ws, L.drv);
  out->kvar = at<double>(ws, L.kvar);
  out->spread = at<double>(ws, L.spread);
  out->qvar = at<double>(ws, L.qvar);
  return TA_OK;
}

namespace {

// Pool and quantise; the status word is cleared first unless a caller that
// runs several plans on one workspace keeps the first error.
ta_status prep_impl(const ta_params* p, const void* Q, const void* K, const void* V, void* ws,
                    size_t ws_bytes, void* stream, bool clear_status) {
  ta_status st = validate(p);
  if (st != TA_OK) return st;
  if ((st = check_tensor(Q)) || (st = check_tensor(K)) || (st = check_tensor(V))) return st;
  if ((st = check_ws(p, ws, ws_bytes)) != TA_OK) return st;
  ta::PlanArgs a;
  fill_plan_args(p, Q, K, V, ws, a);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (clear_status && cudaMemsetAsync(a.status, 0, 4 * sizeof(int32_t), s) != cudaSuccess)
    return TA_ERR_CUDA;
  return ta::launch_prep(a, s) == cudaSuccess ? TA_OK : TA_ERR_CUDA;
}

}  // namespace

ta_status tiered_attn_prep(const ta_params* p, const void* Q, const void* K, const void* V,
                           void* ws, size_t ws_bytes, void* stream) {
  return prep_impl(p, Q, K, V, ws, ws_bytes, stream, true);
}

ta_status tiered_attn_route(const ta_params* p, void* ws, size_t ws_bytes, void* stream) {
  ta_status st = validate(p);
  if (st != TA_OK) return st;
  if ((st = check_ws(p, ws, ws_bytes)) != TA_OK) return st;
  ta::PlanArgs a;
  fill_plan_args(p, nullptr, nullptr, nullptr, ws, a);
  return ta::launch_route(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TA_OK
                                                                                : TA_ERR_CUDA;
}

ta_status tiered_attn_plan(const ta_params* p, const void* Q, const void* K, const void* V,
                           void* ws, size_t ws_bytes, void* stream) {
  ta_status st = tiered_attn_prep(p, Q, K, V, ws, ws_bytes, stream);
  if (st != TA_OK) return st;
  return tiered_attn_route(p, ws, ws_bytes, stream);
}

ta_status tiered_attn_forward(const ta_params* p, const void* Q, const void* K, const void* V,
                              void* ws, size_t ws_bytes, void* O, void* stream) {
  ta_status st = validate(p);
  if (st != TA_OK) return st;
  if ((st = check_tensor(Q)) || (st = check_tensor(K)) || (st = check_tensor(V)) ||
      (st = check_tensor(O)))
    return st;
  if ((st = check_ws(p, ws, ws_bytes)) != TA_OK) return st;
  // native NVFP4 (and residual) tiles are built for d = 128 with 128 x 128 tiles
  const bool fp4 = p->low == TA_LOW_NVFP4 || p->low == TA_LOW_NVFP4_RES;
  if (fp4 && (p->d != 128 || p->block_q != 128 || (p->block_k != 128 && p->block_k != 32)))
    return TA_ERR_UNSUPPORTED;
  const Shape s = shape_of(p);
  const Layout L = layout_of(p);
  ta::AttnArgs a;
  a.B = p->B;
  a.H = p->H;
  a.N = p->N;
  a.d = p->d;
  a.bq = p->block_q;
  a.bk = p->block_k;
  a.low = p->low;
  a.router = p->router;
  a.nQb = (int)s.nQb;
  a.nKb = (int)s.nKb;
  a.sb = p->stride_b;
  a.sh = p->stride_h;
  a.sn = p->stride_n;
  const double scale = p->softmax_scale > 0.0f ? (double)p->softmax_scale : 1.0 / std::sqrt((double)p->d);
  a.scale_log2 = (float)(scale * 1.4426950408889634);
  a.p_offset = p->p_offset_log2;
  a.debug_flags = p->debug_flags;
  a.status = at<int>(ws, L.status);
  a.kbar_b = at<__nv_bfloat16>(ws, L.kbar_b);
  a.vbar_b = at<__nv_bfloat16>(ws, L.vbar_b);
  a.row_counts = at<int>(ws, L.row_counts);
  a.row_lists = at<int>(ws, L.row_lists);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.Np = (int)s.Np;
  a.q_sf = fp4 ? at<uint8_t>(ws, L.q_scales) : nullptr;
  a.k_sf = fp4 ? at<uint8_t>(ws, L.k_scales) : nullptr;
  a.v_sf = fp4 ? at<uint8_t>(ws, L.v_scales) : nullptr;
  a.q_s8 = p->low == TA_LOW_FP8_E4M3 ? at<float>(ws, L.q_scales) : nullptr;
  a.k_s8 = p->low == TA_LOW_FP8_E4M3 ? at<float>(ws, L.k_scales) : nullptr;
  a.v_s8 = p->low == TA_LOW_FP8_E4M3 ? at<float>(ws, L.v_scales) : nullptr;
  a.rq_sf = at<uint8_t>(ws, L.rq_scales);
  a.rk_sf = at<uint8_t>(ws, L.rk_scales);
  a.rv_sf = at<uint8_t>(ws, L.rv_scales);

  CUtensorMap maps[9];
  bool ok = make_map(&maps[0], Q, p->B, p->H, p->N, p->d, p->stride_b, p->stride_h, p->stride_n, p->block_q) &&
            make_map(&maps[1], K, p->B, p->H, p->N, p->d, p->stride_b, p->stride_h, p->stride_n, p->block_k) &&
            make_map(&maps[2], V, p->B, p->H, p->N, p->d, p->stride_b, p->stride_h, p->stride_n, p->block_k);
  // the dequantised copies are contiguous [B*H, N, d]; without a low tier they
  // alias the bf16 inputs (never read)
  if (fp4) {
    const int64_t BH = (int64_t)p->B * p->H;
    ok = ok && make_map_fp4(&maps[3], at<void>(ws, L.q_codes), BH, p->N, p->d / 2, p->block_q) &&
         make_map_fp4(&maps[4], at<void>(ws, L.k_codes), BH, p->N, p->d / 2, p->block_k) &&
         make_map_vt(&maps[5], at<void>(ws, L.v_codes), BH, p->d, s.Np / 2, p->block_k);
    if (p->low == TA_LOW_NVFP4_RES) {
      ok = ok && make_map_fp4(&maps[6], at<void>(ws, L.rq_codes), BH, p->N, p->d / 2, p->block_q) &&
           make_map_fp4(&maps[7], at<void>(ws, L.rk_codes), BH, p->N, p->d / 2, p->block_k) &&
           make_map_vt(&maps[8], at<void>(ws, L.rv_codes), BH, p->d, s.Np / 2, p->block_k);
    } else {
      maps[6] = maps[3];
      maps[7] = maps[4];
      maps[8] = maps[5];
    }
  } else if (p->low == TA_LOW_FP8_E4M3) {
    // FP8 codes, rows of d bytes (128- or 64-byte swizzle)
    const int64_t BH = (int64_t)p->B * p->H;
    ok = ok && make_map_u8(&maps[3], at<void>(ws, L.q_codes), BH, p->N, p->d, p->block_q, p->d) &&
         make_map_u8(&maps[4], at<void>(ws, L.k_codes), BH, p->N, p->d, p->block_k, p->d) &&
         make_map_u8(&maps[5], at<void>(ws, L.v_codes), BH, p->N, p->d, p->block_k, p->d);
  } else {
    maps[3] = maps[0];
    maps[4] = maps[1];
    maps[5] = maps[2];
  }
  if (!fp4) {
    maps[6] = maps[3];  // residual copies: only the NVFP4 + residual format has them
    maps[7] = maps[4];
    maps[8] = maps[5];
  }
  if (!ok) return TA_ERR_CUDA;
  return ta::launch_attn(a, maps, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TA_OK
                                                                                    : TA_ERR_CUDA;
}

ta_status tiered_attn_layer_from_host(const ta_params* p, const void* Qh, const void* Kh,
                                      const void* Vh, void* Oh, void* Qd, void* Kd, void* Vd,
                                      void* Od, void* ws, size_t ws_bytes, void* stream) {
  ta_status st = validate(p);
  if (st != TA_OK) return st;
  if (!Qh || !Kh || !Vh || !Oh) return TA_ERR_INVALID_ARG;
  if ((st = check_tensor(Qd)) || (st = check_tensor(Kd)) || (st = check_tensor(Vd)) ||
      (st = check_tensor(Od)))
    return st;
  if ((st = check_ws(p, ws, ws_bytes)) != TA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t head = (int64_t)p->N * p->d;   // elements of one (b, h) slice
  const bool packed = p->stride_n == p->d && p->stride_h == head && p->stride_b == (int64_t)p->H * head;
  const int64_t BH = (int64_t)p->B * p->H;
  if (!packed || BH < 2) {
    // one chunk, all on the caller's stream
    const int64_t span = (int64_t)(p->B - 1) * p->stride_b + (int64_t)(p->H - 1) * p->stride_h +
                         (int64_t)(p->N - 1) * p->stride_n + p->d;
    const size_t bytes = (size_t)span * 2;
    if (cudaMemcpyAsync(Qd, Qh, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(Kd, Kh, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(Vd, Vh, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return TA_ERR_CUDA;
    if ((st = tiered_attn_plan(p, Qd, Kd, Vd, ws, ws_bytes, stream)) != TA_OK) return st;
    if ((st = tiered_attn_forward(p, Qd, Kd, Vd, ws, ws_bytes, Od, stream)) != TA_OK) return st;
    if (cudaMemcpyAsync(Oh, Od, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return TA_ERR_CUDA;
    return TA_OK;
  }

  // Packed heads: the layer runs in chunks of consecutive (b, h) slices (every
  // head is independent), so that the copy of chunk c+1 in, the attention of
  // chunk c and the copy of chunk c-1 out overlap.  Copies in go on one
  // library stream, copies out on another, the kernels on the caller's
  // stream; events order them, and the caller's stream waits for the last
  // copy out.
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TA_ERR_CUDA;
  std::lock_guard<std::mutex> guard(g_copy_mu);
  CopyStreams& cs = g_copy[dev];
  if (!cs.ready) {
    if (cudaStreamCreateWithFlags(&cs.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&cs.out, cudaStreamNonBlocking) != cudaSuccess)
      return TA_ERR_CUDA;
    for (auto& e : cs.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return TA_ERR_CUDA;
    cs.ready = true;
  }
  const int nch = (int)(BH < kChunks ? BH : kChunks);
  cudaEvent_t ev_entry = cs.ev[0], ev_done = cs.ev[1];
  cudaEvent_t* ev_in = cs.ev + 2;
  cudaEvent_t* ev_out = cs.ev + 2 + kChunks;
  // every earlier use of the device buffers on the caller's stream comes first
  if (cudaEventRecord(ev_entry, s) != cudaSuccess || cudaStreamWaitEvent(cs.in, ev_entry, 0) != cudaSuccess)
    return TA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return TA_ERR_CUDA;  // status
  auto chunk = [&](int c, int64_t& bh0, int64_t& n) {
    bh0 = BH * c / nch;
    n = BH * (c + 1) / nch - bh0;
  };
  const char* qh = static_cast<const char*>(Qh);
  const char* kh = static_cast<const char*>(Kh);
  const char* vh = static_cast<const char*>(Vh);
  char* oh = static_cast<char*>(Oh);
  char* qd = static_cast<char*>(Qd);
  char* kd = static_cast<char*>(Kd);
  char* vd = static_cast<char*>(Vd);
  char* od = static_cast<char*>(Od);
  for (int c = 0; c < nch; ++c) {
    int64_t bh0, n;
    chunk(c, bh0, n);
    const size_t off = (size_t)bh0 * head * 2, bytes = (size_t)n * head * 2;
    if (cudaMemcpyAsync(qd + off, qh + off, bytes, cudaMemcpyHostToDevice, cs.in) != cudaSuccess ||
        cudaMemcpyAsync(kd + off, kh + off, bytes, cudaMemcpyHostToDevice, cs.in) != cudaSuccess ||
        cudaMemcpyAsync(vd + off, vh + off, bytes, cudaMemcpyHostToDevice, cs.in) != cudaSuccess ||
        cudaEventRecord(ev_in[c], cs.in) != cudaSuccess)
      return TA_ERR_CUDA;
  }
  for (int c = 0; c < nch; ++c) {
    int64_t bh0, n;
    chunk(c, bh0, n);
    const size_t off = (size_t)bh0 * head * 2, bytes = (size_t)n * head * 2;
    ta_params pc = *p;   // the chunk as a layer of one batch of n heads
    pc.B = 1;
    pc.H = (int32_t)n;
    pc.stride_b = (int64_t)n * head;
    if (cudaStreamWaitEvent(s, ev_in[c], 0) != cudaSuccess) return TA_ERR_CUDA;
    if ((st = prep_impl(&pc, qd + off, kd + off, vd + off, ws, ws_bytes, stream, false)) != TA_OK ||
        (st = tiered_attn_route(&pc, ws, ws_bytes, stream)) != TA_OK ||
        (st = tiered_attn_forward(&pc, qd + off, kd + off, vd + off, ws, ws_bytes, od + off, stream)) != TA_OK)
      return st;
    if (cudaEventRecord(ev_out[c], s) != cudaSuccess || cudaStreamWaitEvent(cs.out, ev_out[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + off, od + off, bytes, cudaMemcpyDeviceToHost, cs.out) != cudaSuccess)
      return TA_ERR_CUDA;
  }
  if (cudaEventRecord(ev_done, cs.out) != cudaSuccess || cudaStreamWaitEvent(s, ev_done, 0) != cudaSuccess)
    return TA_ERR_CUDA;
  return TA_OK;
}

ta_status tiered_attn_get_status(const void* ws, void* stream) {
  if (!ws || !aligned(ws, kAlign)) return TA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return TA_ERR_CUDA;
  int32_t st[4] = {0, 0, 0, 0};
  if (cudaMemcpy(st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return TA_ERR_CUDA;
  return static_cast<ta_status>(st[0]);
}

}  // extern "C"
