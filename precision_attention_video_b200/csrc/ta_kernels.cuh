// ta_kernels.cuh -- argument blocks and launchers of the tiered-attention
// kernels (router / quantiser / fused attention), shared by the C ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tiered_attn.h"

namespace ta {

// Everything the plan stage reads and writes (device pointers into the
// workspace; null where the low format does not produce the array).
struct PlanArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t sb, sh, sn;           // element strides of Q, K, V
  int B, H, N, d, bq, bk, low;  // shape, tiles, ta_low_format
  int R;                        // rows per prep chunk = max(bq, bk)
  int nQb, nKb, Np;             // ceil(N/bq), ceil(N/bk), 16*ceil(N/16)
  int n_tau;
  double tau[3];
  int keep_diag;
  int router;                   // ta_router
  double price;                 // TA_ROUTER_PRICE's price
  double cost[4];               // TA_ROUTER_PRICE's tier costs by tier code (defaults resolved)
  double retention;             // TA_ROUTER_ENTROPY's kappa
  double scale;                 // softmax scale (fp64 in the router)
  int* status;
  double* qbar;
  double* kbar;
  __nv_bfloat16* kbar_b;
  __nv_bfloat16* vbar_b;
  int* n_k;
  double* logits;
  double* mass;
  double* kvar;                 // [BH, nKb, d] key-block coordinate variances (price router)
  double* qvar;                 // [BH, nQb, d] query-block coordinate variances (price router)
  double* spread;               // [BH, nQb, nKb] skip error factor delta (price router)
  uint8_t* tier_map;
  int* row_counts;
  int* row_lists;
  uint8_t *q_codes, *k_codes, *v_codes;
  void *q_scales, *k_scales, *v_scales;
  uint8_t *rq_codes, *rk_codes, *rv_codes;
  uint8_t *rq_scales, *rk_scales, *rv_scales;
};

// Fused attention arguments.
struct AttnArgs {
  int B, H, N, d, bq, bk, low;
  int router;                   // ta_router of the plan (selects the kernel)
  int nQb, nKb;
  int64_t sb, sh, sn;           // element strides of Q and O
  float scale_log2;             // softmax_scale * log2(e)
  int p_offset;                 // o of P' = 2^o exp(s - m)
  int debug_flags;
  int* status;
  const __nv_bfloat16* Q;       // queries [B, H, N, d] (strides sb, sh, sn)
  const __nv_bfloat16* kbar_b;  // skip pseudo-keys [BH, nKb, d]
  const __nv_bfloat16* vbar_b;
  const int* row_counts;
  const int* row_lists;
  __nv_bfloat16* O;
  // NVFP4 scales of the low copies (used by the native FP4 tile path):
  // Q, K [BH, N, d/16]; V [BH, Np/16, d]
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  // scales of the residual NVFP4 copies (TA_LOW_NVFP4_RES), same layouts
  const uint8_t* rq_sf;
  const uint8_t* rk_sf;
  const uint8_t* rv_sf;
  // per-tile power-of-two scales of the FP8 copies: Q [BH, nQb], K / V [BH, nKb]
  const float* q_s8;
  const float* k_s8;
  const float* v_s8;
  int Np;
};

cudaError_t launch_prep(const PlanArgs& a, cudaStream_t s);
cudaError_t launch_route(const PlanArgs& a, cudaStream_t s);
cudaError_t launch_attn(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t s);
// The two-group kernel (d = 128, 128 x 128 tiles); cudaErrorNotSupported for
// other shapes.
cudaError_t launch_attn2(const AttnArgs& a, const CUtensorMap* maps, cudaStream_t s);

}  // namespace ta
