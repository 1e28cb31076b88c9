// ta_route.cu -- the router: pooled block logits, pooled block softmax,
// cumulative-mass (or single-price) tiers and compacted per-row tile lists.
//
// "Triage" (zhuanzhiai paper page, abstract) predicts each tile's treatment
// from block statistics; "HierPAS" (conference listing, abstract) estimates the
// attention pattern cheaply and keeps precision where the mass is; "APT"
// (Lattice paper summary, APDT) turns attention probability into selection and
// precision with two thresholds.  Per head and query block i:
//   sbar_ij = (qbar_i . kbar_j) * scale,
//   M_ij    = n_j exp(sbar_ij - max_j sbar_ij) / sum_j (.),
//   sort j by (-M_ij, j); C_r = exclusive prefix sum of the sorted masses;
//   tier(rank r) = the most precise tier t with C_r < tau_t, else skip;
//   key blocks meeting query block i's token range become full;
//   list = full blocks, then residual, low, skip; within a tier in (-M, j)
//   order, so a query block meets its heaviest key blocks first.
// The entropy router ("HierPAS" abstract: retention ratios from an entropy
// analysis of a cheap pattern estimate) keeps, per query block, the
// ceil(kappa exp(H)) heaviest key blocks, H the entropy of the pooled row.
// The price router ("Triage" abstract: move a tile to a more accurate tier
// only when its predicted error reduction is worth the extra compute at a
// single price) gives each tile the tier of least M * eps_t + price * cost_t,
// with the skip tier's eps the block's logit spread delta (see price_tier).
// The router runs in fp64 end to end (means, logits, exp, prefix), so its
// cumulative masses agree with an fp64 evaluation to ~1e-15 relative and the
// tier map only depends on the ordering rule, not on rounding.
#include "ta_common.cuh"
#include "ta_kernels.cuh"

namespace ta {
namespace {

// ---------------------------------------------------------------------------
// Pooled logits: logits[bh, i, j] = scale * sum_c qbar[bh, i, c] kbar[bh, j, c]
// and, for the price router, the skip tier's error factor
// spread[bh, i, j] = scale * sqrt(sum_c (qbar[bh, i, c]^2 + qvar[bh, i, c]) kvar[bh, j, c]).
// 32 x 32 output tile per CTA, 2 x 2 per thread, d staged 32 at a time.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) logits_kernel(const PlanArgs a) {
  __shared__ double qs[32][33];
  __shared__ double ks[32][33];
  __shared__ double vs[32][33];
  __shared__ double qw[32][33];   // qbar^2 + qvar (price router)
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int bh = blockIdx.z, i0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  const int D = a.d;
  const double* qb = a.qbar + (int64_t)bh * a.nQb * D;
  const double* kb = a.kbar + (int64_t)bh * a.nKb * D;
  const double* kvb = a.kvar ? a.kvar + (int64_t)bh * a.nKb * D : nullptr;
  const double* qvb = a.qvar ? a.qvar + (int64_t)bh * a.nQb * D : nullptr;
  double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
  double spr[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
  for (int c0 = 0; c0 < D; c0 += 32) {
    for (int e = tid; e < 32 * 32; e += 256) {
      const int r = e / 32, c = e % 32;
      qs[r][c] = (i0 + r < a.nQb) ? qb[(int64_t)(i0 + r) * D + c0 + c] : 0.0;
      ks[r][c] = (j0 + r < a.nKb) ? kb[(int64_t)(j0 + r) * D + c0 + c] : 0.0;
      if (kvb) {
        vs[r][c] = (j0 + r < a.nKb) ? kvb[(int64_t)(j0 + r) * D + c0 + c] : 0.0;
        qw[r][c] = (i0 + r < a.nQb) ? qs[r][c] * qs[r][c] + qvb[(int64_t)(i0 + r) * D + c0 + c] : 0.0;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      const double q0 = qs[ty * 2][c], q1 = qs[ty * 2 + 1][c];
      const double k0 = ks[tx * 2][c], k1 = ks[tx * 2 + 1][c];
      acc[0][0] += q0 * k0;
      acc[0][1] += q0 * k1;
      acc[1][0] += q1 * k0;
      acc[1][1] += q1 * k1;
    }
    if (kvb) {
#pragma unroll 8
      for (int c = 0; c < 32; ++c) {
        const double w0 = qw[ty * 2][c], w1 = qw[ty * 2 + 1][c];
        const double v0 = vs[tx * 2][c], v1 = vs[tx * 2 + 1][c];
        spr[0][0] += w0 * v0;
        spr[0][1] += w0 * v1;
        spr[1][0] += w1 * v0;
        spr[1][1] += w1 * v1;
      }
    }
    __syncthreads();
  }
  for (int u = 0; u < 2; ++u)
    for (int v = 0; v < 2; ++v) {
      const int i = i0 + ty * 2 + u, j = j0 + tx * 2 + v;
      if (i < a.nQb && j < a.nKb) {
        a.logits[((int64_t)bh * a.nQb + i) * a.nKb + j] = acc[u][v] * a.scale;
        if (kvb) a.spread[((int64_t)bh * a.nQb + i) * a.nKb + j] = a.scale * sqrt(spr[u][v]);
      }
    }
}

// The price router's tier of one tile: the least predicted error + price *
// cost among the tiers the low format provides, cheapest first, keeping the
// cheaper tier on a tie.  Error = M * eps (eps: the tier's unit roundoff; for
// skip, the tile's spread delta); cost = the tier's per-tile time (ta_params
// tier_cost, by default as measured on the fused kernel).
__device__ __forceinline__ int price_tier(double M, double delta, double price, int low,
                                          double c_skip, double c_low, double c_res, double c_full) {
  int best = TA_TIER_SKIP;
  double obj = M * delta + price * c_skip;
  auto consider = [&](int tier, double eps, double cost) {
    const double o = M * eps + price * cost;
    if (o < obj) {
      obj = o;
      best = tier;
    }
  };
  if (low == TA_LOW_FP8_E4M3) consider(TA_TIER_LOW, 0.0625, c_low);
  if (low == TA_LOW_NVFP4 || low == TA_LOW_NVFP4_RES) consider(TA_TIER_LOW, 0.25, c_low);
  if (low == TA_LOW_NVFP4_RES) consider(TA_TIER_RES, 0.0625, c_res);
  consider(TA_TIER_FULL, 0.00390625, c_full);
  return best;
}

// ---------------------------------------------------------------------------
// Per-row routing, one warp per (bh, query block).
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 8;

__device__ __forceinline__ bool before(double ka, int ia, double kb, int ib) {
  return (ka > kb) || (ka == kb && ia < ib);
}

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Bitonic sort of 32*E (key, idx) pairs held by one warp, element e = k*32 +
// lane in register k of lane `lane`, into (-key, idx) order.  Partners less
// than 32 apart are in other lanes (shuffles); farther ones are in this lane's
// registers.  Fully unrolled, so every register index is a constant.
template <int E>
__device__ __forceinline__ void warp_sort(double (&key)[E], int (&idx)[E], int lane) {
  constexpr int n = 32 * E;
#pragma unroll
  for (int size = 2; size <= n; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {
        const int ks = stride / 32;
#pragma unroll
        for (int k = 0; k < E; ++k) {
          const int kp = k ^ ks;
          if (kp > k) {
            const bool up = (((k * 32 + lane) & size) == 0);
            const bool sw = up ? before(key[kp], idx[kp], key[k], idx[k])
                               : before(key[k], idx[k], key[kp], idx[kp]);
            if (sw) {
              const double tk = key[k];
              key[k] = key[kp];
              key[kp] = tk;
              const int ti = idx[k];
              idx[k] = idx[kp];
              idx[kp] = ti;
            }
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < E; ++k) {
          const double ok = __shfl_xor_sync(0xffffffffu, key[k], stride);
          const int oi = __shfl_xor_sync(0xffffffffu, idx[k], stride);
          const bool lower = (lane & stride) == 0;
          const bool up = (((k * 32 + lane) & size) == 0);
          // the lower position of an ascending pair keeps the element that
          // comes first; of a descending pair, the one that comes second
          const bool mine_first = before(key[k], idx[k], ok, oi);
          if ((lower == up) != mine_first) {
            key[k] = ok;
            idx[k] = oi;
          }
        }
      }
    }
  }
}

template <int E>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(const PlanArgs a) {
  constexpr int sortn = 32 * E;
  __shared__ uint8_t tier_s[kRouteWarps][sortn];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint8_t* tier = tier_s[warp];

  const int64_t g = (int64_t)blockIdx.x * kRouteWarps + warp;  // global row
  const int64_t nrows = (int64_t)a.B * a.H * a.nQb;
  if (g >= nrows) return;
  const int i = (int)(g % a.nQb);
  const int nKb = a.nKb;
  const double* lrow = a.logits + g * nKb;

  // pooled block softmax weighted by key counts; element e = k*32 + lane
  double key[E];
  int idx[E];
  double mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int j = k * 32 + lane;
    key[k] = j < nKb ? lrow[j] : -INFINITY;
    mx = fmax(mx, key[k]);
  }
  mx = warp_max(mx);
  double part = 0.0;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int j = k * 32 + lane;
    if (j < nKb) {
      const int nj = min(a.bk, a.N - j * a.bk);
      key[k] = (double)nj * exp(key[k] - mx);
      part += key[k];
    }
  }
  const double total = warp_sum(part);
  // entropy router: keep the ceil(kappa exp(H)) heaviest blocks of the row
  int keep = nKb;
  if (a.router == TA_ROUTER_ENTROPY) {
    double hp = 0.0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int j = k * 32 + lane;
      if (j < nKb) {
        const double m = key[k] / total;
        if (m > 0.0) hp -= m * log(m);
      }
    }
    const double want = a.retention * exp(warp_sum(hp));
    keep = (int)fmin((double)nKb, fmax(1.0, ceil(want)));
  }
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int j = k * 32 + lane;
    if (j < nKb) {
      const double m = key[k] / total;
      key[k] = m;
      idx[k] = j;
      a.mass[g * nKb + j] = m;
      if (a.router == TA_ROUTER_PRICE)
        tier[j] = (uint8_t)price_tier(m, a.spread[g * nKb + j], a.price, a.low, a.cost[TA_TIER_SKIP],
                                      a.cost[TA_TIER_LOW], a.cost[TA_TIER_RES], a.cost[TA_TIER_FULL]);
    } else {
      key[k] = -1.0;
      idx[k] = 0x7fffffff - (sortn - j);
    }
  }

  // sort into (-M, j) order: rank r = k*32 + lane holds (key[k], idx[k])
  warp_sort<E>(key, idx, lane);

  // tiers by rank: exclusive prefix of the sorted masses, rank r = k*32 + lane
  int codes[3];
  if (a.n_tau == 1) {
    codes[0] = TA_TIER_FULL;
  } else if (a.n_tau == 2) {
    codes[0] = TA_TIER_FULL;
    codes[1] = TA_TIER_LOW;
  } else {
    codes[0] = TA_TIER_FULL;
    codes[1] = TA_TIER_RES;
    codes[2] = TA_TIER_LOW;
  }
  if (a.router != TA_ROUTER_PRICE) {
    const int kept_low = codes[a.n_tau - 1];   // least precise kept tier
    double base = 0.0;                          // masses of all ranks before this row of 32
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const double mk = fmax(key[k], 0.0);
      double incl = mk;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const double C = base + (incl - mk);
      base += __shfl_sync(0xffffffffu, incl, 31);
      const int j = idx[k], r = k * 32 + lane;
      if (j < nKb) {
        int t = TA_TIER_SKIP;
        for (int q = a.n_tau - 1; q >= 0; --q)
          if (C < a.tau[q]) t = codes[q];
        if (a.router == TA_ROUTER_ENTROPY) t = (r >= keep) ? TA_TIER_SKIP : (t == TA_TIER_SKIP ? kept_low : t);
        tier[j] = (uint8_t)t;
      }
    }
  }
  __syncwarp();
  if (a.keep_diag && lane == 0) {
    const int r0 = i * a.bq, r1 = min(a.N, (i + 1) * a.bq);
    for (int j = r0 / a.bk; j <= (r1 - 1) / a.bk; ++j) tier[j] = TA_TIER_FULL;
  }
  __syncwarp();

  // tier map row, counts and the compacted list: tiers in the order full,
  // res, low, skip; within a tier the blocks keep their (-M, j) rank order
  for (int j = lane; j < nKb; j += 32) a.tier_map[g * nKb + j] = tier[j];
  const int order[4] = {TA_TIER_FULL, TA_TIER_RES, TA_TIER_LOW, TA_TIER_SKIP};
  int base = 0;
  for (int q = 0; q < 4; ++q) {
    const int t = order[q];
    int cnt = 0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int j = idx[k];
      const bool p = (j < nKb) && tier[j] == t;
      const unsigned bal = __ballot_sync(0xffffffffu, p);
      if (p) a.row_lists[g * nKb + base + cnt + __popc(bal & ((1u << lane) - 1u))] = j;
      cnt += __popc(bal);
    }
    if (lane == 0) a.row_counts[g * 4 + q] = cnt;
    base += cnt;
  }
}

}  // namespace

cudaError_t launch_route(const PlanArgs& a, cudaStream_t s) {
  dim3 g1((a.nQb + 31) / 32, (a.nKb + 31) / 32, a.B * a.H);
  logits_kernel<<<g1, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int sortn = 32;
  while (sortn < a.nKb) sortn <<= 1;
  const int64_t rows = (int64_t)a.B * a.H * a.nQb;
  dim3 g2((unsigned)((rows + kRouteWarps - 1) / kRouteWarps));
  switch (sortn) {
    case 32: route_kernel<1><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 64: route_kernel<2><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 128: route_kernel<4><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 256: route_kernel<8><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 512: route_kernel<16><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 1024: route_kernel<32><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ta
