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
// 128 x 128 output tile per CTA, 8 x 8 per thread (rows ty + 16 u, columns
// tx + 16 v, so that a warp's 16 tx read 16 consecutive doubles: no bank
// conflicts), d staged kLC coordinates at a time into two alternating
// buffers (the next chunk's global loads overlap this chunk's FMAs); 16
// shared loads feed 64 fp64 FMAs.  The spread is a second pass over d with
// the same registers.
// ---------------------------------------------------------------------------
constexpr int kLT = 128, kLC = 8;

template <bool SPREAD>
__device__ __forceinline__ void logits_pass(const PlanArgs& a, int bh, int i0, int j0, double (&qs)[2][kLC][kLT],
                                            double (&ks)[2][kLC][kLT], double (&acc)[8][8]) {
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int D = a.d;
  const double* qb = a.qbar + (int64_t)bh * a.nQb * D;
  const double* kb = (SPREAD ? a.kvar : a.kbar) + (int64_t)bh * a.nKb * D;
  const double* qvb = SPREAD ? a.qvar + (int64_t)bh * a.nQb * D : nullptr;
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[u][v] = 0.0;
  // each thread stages elements e = tid + 256 w (w < kStage) of the 128 rows x
  // kLC coordinates of both operands: r = e / kLC, c = e % kLC
  constexpr int kStage = kLT * kLC / 256;
  double pq[kStage], pk[kStage];
  auto fetch = [&](int c0) {
#pragma unroll
    for (int w = 0; w < kStage; ++w) {
      const int e = tid + 256 * w, r = e / kLC, c = e % kLC;
      const bool qi = i0 + r < a.nQb, kj = j0 + r < a.nKb;
      double q = qi ? qb[(int64_t)(i0 + r) * D + c0 + c] : 0.0;
      if (SPREAD && qi) q = q * q + qvb[(int64_t)(i0 + r) * D + c0 + c];
      pq[w] = q;
      pk[w] = kj ? kb[(int64_t)(j0 + r) * D + c0 + c] : 0.0;
    }
  };
  fetch(0);
  for (int c0 = 0, buf = 0; c0 < D; c0 += kLC, buf ^= 1) {
#pragma unroll
    for (int w = 0; w < kStage; ++w) {
      const int e = tid + 256 * w, r = e / kLC, c = e % kLC;
      qs[buf][c][r] = pq[w];
      ks[buf][c][r] = pk[w];
    }
    __syncthreads();
    // the next chunk's loads are in flight while this one is multiplied; the
    // buffer written next was last read before the barrier above
    if (c0 + kLC < D) fetch(c0 + kLC);
#pragma unroll 2
    for (int c = 0; c < kLC; ++c) {
      double q[8], k[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = qs[buf][c][ty + 16 * u];
#pragma unroll
      for (int v = 0; v < 8; ++v) k[v] = ks[buf][c][tx + 16 * v];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = fma(q[u], k[v], acc[u][v]);
    }
  }
  __syncthreads();   // the caller's next pass restages both buffers
}

__global__ void __launch_bounds__(256) logits_kernel(const PlanArgs a) {
  __shared__ double qs[2][kLC][kLT];
  __shared__ double ks[2][kLC][kLT];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int bh = blockIdx.z, i0 = blockIdx.x * kLT, j0 = blockIdx.y * kLT;
  double acc[8][8];
  logits_pass<false>(a, bh, i0, j0, qs, ks, acc);
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
      if (i < a.nQb && j < a.nKb) a.logits[((int64_t)bh * a.nQb + i) * a.nKb + j] = acc[u][v] * a.scale;
    }
  if (a.kvar) {
    logits_pass<true>(a, bh, i0, j0, qs, ks, acc);
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
        if (i < a.nQb && j < a.nKb) a.spread[((int64_t)bh * a.nQb + i) * a.nKb + j] = a.scale * sqrt(acc[u][v]);
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

// ---------------------------------------------------------------------------
// Per-row routing for long rows (more than 256 key blocks), one CTA per
// (bh, query block): the same steps as route_kernel, with the row held in
// shared memory and the (-M, j) sort, the exclusive prefix of the sorted
// masses and the list compaction done by the whole CTA.  A warp with 32
// elements a lane (route_kernel<32>) needs 159 registers and runs one CTA
// per SM; here many rows are in flight on each SM.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 256;

// Block-wide exclusive prefix sum of one value per thread; `total` gets the sum.
__device__ __forceinline__ double block_excl_scan(double v, double* wsum, double& total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  double base = 0.0, tot = 0.0;
  for (int w = 0; w < kRowThreads / 32; ++w) {
    const double x = wsum[w];
    if (w < warp) base += x;
    tot += x;
  }
  __syncthreads();
  total = tot;
  return base + incl - v;
}
__device__ __forceinline__ int block_excl_scan_int(int v, int* wsum, int& total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = 0, tot = 0;
  for (int w = 0; w < kRowThreads / 32; ++w) {
    const int x = wsum[w];
    if (w < warp) base += x;
    tot += x;
  }
  __syncthreads();
  total = tot;
  return base + incl - v;
}
__device__ __forceinline__ double block_reduce(double v, double* wsum, bool is_max) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmax(v, y) : v + y;
  }
  if (lane == 0) wsum[warp] = v;
  __syncthreads();
  double r = is_max ? -INFINITY : 0.0;
  for (int w = 0; w < kRowThreads / 32; ++w) r = is_max ? fmax(r, wsum[w]) : r + wsum[w];
  __syncthreads();
  return r;
}

// Sort key of key block j with pooled mass m >= 0: the float of m rounded
// toward zero (so that a larger float means a larger mass) in the high word,
// complemented so that ascending keys run by descending mass, and j in the
// low word (lower j first among equal floats).  Blocks whose masses round to
// the same float are put in exact (-M, j) order afterwards (fix_exact_order).
__device__ __forceinline__ uint64_t sort_key(double m, int j) {
  const uint32_t hi = ~__float_as_uint(__double2float_rz(m));
  return ((uint64_t)hi << 32) | (uint32_t)j;
}

// Bitonic sort, ascending, of kRowThreads * EPT distinct 64-bit keys; thread
// tid holds positions tid * EPT .. tid * EPT + EPT - 1.  The network is
// unrolled: strides below EPT run inside a thread, strides below 32 * EPT
// between the lanes of a warp (shuffles), longer ones through shared memory
// (`xk`: one key per thread and slot, slot-major so that a warp's accesses
// fall on distinct banks).
template <int EPT>
__device__ __forceinline__ void sort_row(uint64_t (&kr)[EPT], uint64_t* xk) {
  constexpr int sortn = kRowThreads * EPT;
  constexpr int kLog = (sortn == 512) ? 9 : 10;
  static_assert((1 << kLog) == sortn, "sort width");
  const int tid = threadIdx.x;
#pragma unroll
  for (int ls = 1; ls <= kLog; ++ls) {
#pragma unroll
    for (int lt = ls - 1; lt >= 0; --lt) {
      const int size = 1 << ls, stride = 1 << lt;
      if (stride < EPT) {
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          if (e & stride) continue;
          const bool up = ((tid * EPT + e) & size) == 0;
          const uint64_t lo = kr[e] < kr[e + stride] ? kr[e] : kr[e + stride];
          const uint64_t hi = kr[e] < kr[e + stride] ? kr[e + stride] : kr[e];
          kr[e] = up ? lo : hi;
          kr[e + stride] = up ? hi : lo;
        }
        continue;
      }
      // the partner of position p = tid * EPT + e is p ^ stride = (tid ^ m) * EPT + e;
      // the lower position of an ascending pair keeps the smaller key
      const int m = stride / EPT;
      const bool keep_min = ((tid & m) == 0) == (((tid * EPT) & size) == 0);
      uint64_t kp[EPT];
      if (stride < 32 * EPT) {
#pragma unroll
        for (int e = 0; e < EPT; ++e) kp[e] = __shfl_xor_sync(0xffffffffu, kr[e], m);
      } else {
#pragma unroll
        for (int e = 0; e < EPT; ++e) xk[e * kRowThreads + tid] = kr[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < EPT; ++e) kp[e] = xk[e * kRowThreads + (tid ^ m)];
        __syncthreads();
      }
#pragma unroll
      for (int e = 0; e < EPT; ++e) kr[e] = ((kp[e] < kr[e]) == keep_min) ? kp[e] : kr[e];
    }
  }
}

// After sort_row the order is exact except, possibly, among blocks whose
// masses round to one float (ordered there by j alone).  Ranks r and r + 1
// out of (-M, j) order are looked for over the whole row; if any is found
// (rare: masses within 2^-24 of each other), one thread reorders the row's
// nKb ranks by insertion, which costs one pass plus the few moves.  `xi`
// holds the block of each rank on return; `mass` the exact masses by block.
template <int EPT>
__device__ __forceinline__ void fix_exact_order(const uint64_t (&kr)[EPT], int* xi, const double* mass,
                                                int nKb) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int e = 0; e < EPT; ++e) xi[tid * EPT + e] = (int)(uint32_t)kr[e];
  __syncthreads();
  bool bad = false;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int r = tid * EPT + e;
    if (r + 1 < nKb) {
      const int ja = xi[r], jb = xi[r + 1];
      bad |= !before(mass[ja], ja, mass[jb], jb);
    }
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      for (int r = 1; r < nKb; ++r) {
        const int j = xi[r];
        const double mj = mass[j];
        int q = r - 1;
        while (q >= 0 && before(mj, j, mass[xi[q]], xi[q])) {
          xi[q + 1] = xi[q];
          --q;
        }
        xi[q + 1] = j;
      }
    }
    __syncthreads();
  }
}

// EPT: elements a thread owns (sortn = kRowThreads * EPT, a power of two).
// Thread tid owns key blocks tid * EPT .. (contiguous) before the sort and
// ranks tid * EPT .. after it, which makes the prefix over the sorted masses
// a scan over threads.
template <int EPT>
__global__ void __launch_bounds__(kRowThreads) route_row_kernel(const PlanArgs a) {
  constexpr int sortn = kRowThreads * EPT;
  __shared__ uint64_t xk[sortn];
  __shared__ int xi[sortn];
  __shared__ double mass_s[sortn];
  __shared__ uint8_t tier[sortn];
  __shared__ double wsum_d[kRowThreads / 32];
  __shared__ int wsum_i[kRowThreads / 32];
  const int tid = threadIdx.x;
  const int64_t g = blockIdx.x;   // global row (bh, i)
  const int i = (int)(g % a.nQb);
  const int nKb = a.nKb;
  const double* lrow = a.logits + g * nKb;

  // pooled block softmax weighted by key counts
  double kr[EPT];
  int ir[EPT];
  double mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int j = tid * EPT + e;
    kr[e] = j < nKb ? lrow[j] : -INFINITY;
    mx = fmax(mx, kr[e]);
  }
  mx = block_reduce(mx, wsum_d, true);
  double part = 0.0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int j = tid * EPT + e;
    if (j < nKb) {
      const int nj = min(a.bk, a.N - j * a.bk);
      kr[e] = (double)nj * exp(kr[e] - mx);
      part += kr[e];
    }
  }
  const double total = block_reduce(part, wsum_d, false);
  int keep = nKb;
  if (a.router == TA_ROUTER_ENTROPY) {
    double hp = 0.0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int j = tid * EPT + e;
      if (j < nKb) {
        const double m = kr[e] / total;
        if (m > 0.0) hp -= m * log(m);
      }
    }
    const double want = a.retention * exp(block_reduce(hp, wsum_d, false));
    keep = (int)fmin((double)nKb, fmax(1.0, ceil(want)));
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int j = tid * EPT + e;
    if (j < nKb) {
      const double m = kr[e] / total;
      kr[e] = m;
      ir[e] = j;
      mass_s[j] = m;
      a.mass[g * nKb + j] = m;
      if (a.router == TA_ROUTER_PRICE)
        tier[j] = (uint8_t)price_tier(m, a.spread[g * nKb + j], a.price, a.low, a.cost[TA_TIER_SKIP],
                                      a.cost[TA_TIER_LOW], a.cost[TA_TIER_RES], a.cost[TA_TIER_FULL]);
    } else {
      kr[e] = -1.0;
      ir[e] = 0x7fffffff - (sortn - j);
    }
  }

  // rank order: padding (keys above every real block's) sorts last
  uint64_t key[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) key[e] = ir[e] < nKb ? sort_key(kr[e], ir[e]) : (~0ull - (uint64_t)(sortn - tid * EPT - e));
  sort_row<EPT>(key, xk);
  fix_exact_order<EPT>(key, xi, mass_s, nKb);
  // rank tid * EPT + e now holds block ir[e] with mass kr[e]
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int r = tid * EPT + e;
    ir[e] = r < nKb ? xi[r] : 0x7fffffff;
    kr[e] = r < nKb ? mass_s[ir[e]] : -1.0;
  }

  // tiers by rank: exclusive prefix C of the sorted masses
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
    const int kept_low = codes[a.n_tau - 1];
    double mine = 0.0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) mine += fmax(kr[e], 0.0);
    double tot;
    double C = block_excl_scan(mine, wsum_d, tot);
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int r = tid * EPT + e;
      const int j = ir[e];
      const double mk = fmax(kr[e], 0.0);
      if (j < nKb) {
        int t = TA_TIER_SKIP;
        for (int q = a.n_tau - 1; q >= 0; --q)
          if (C < a.tau[q]) t = codes[q];
        if (a.router == TA_ROUTER_ENTROPY) t = (r >= keep) ? TA_TIER_SKIP : (t == TA_TIER_SKIP ? kept_low : t);
        tier[j] = (uint8_t)t;
      }
      C += mk;
    }
  }
  __syncthreads();
  if (a.keep_diag && tid == 0) {
    const int r0 = i * a.bq, r1 = min(a.N, (i + 1) * a.bq);
    for (int j = r0 / a.bk; j <= (r1 - 1) / a.bk; ++j) tier[j] = TA_TIER_FULL;
  }
  __syncthreads();

  // tier map row, counts and the compacted list (tiers full, res, low, skip;
  // within a tier in rank order)
  for (int j = tid; j < nKb; j += kRowThreads) a.tier_map[g * nKb + j] = tier[j];
  uint8_t tr[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) tr[e] = ir[e] < nKb ? tier[ir[e]] : 0xFF;
  const int order[4] = {TA_TIER_FULL, TA_TIER_RES, TA_TIER_LOW, TA_TIER_SKIP};
  int base = 0;
  for (int q = 0; q < 4; ++q) {
    const int t = order[q];
    int mine = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) mine += (tr[e] == t) ? 1 : 0;
    int cnt;
    int pos = block_excl_scan_int(mine, wsum_i, cnt);
#pragma unroll
    for (int e = 0; e < EPT; ++e)
      if (tr[e] == t) a.row_lists[g * nKb + base + pos++] = ir[e];
    if (tid == 0) a.row_counts[g * 4 + q] = cnt;
    base += cnt;
  }
}

}  // namespace

cudaError_t launch_route(const PlanArgs& a, cudaStream_t s) {
  dim3 g1((a.nQb + kLT - 1) / kLT, (a.nKb + kLT - 1) / kLT, a.B * a.H);
  logits_kernel<<<g1, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int sortn = 32;
  while (sortn < a.nKb) sortn <<= 1;
  const int64_t rows = (int64_t)a.B * a.H * a.nQb;
  dim3 g2((unsigned)((rows + kRouteWarps - 1) / kRouteWarps));
  // rows of up to 256 key blocks: one warp a row; longer rows: one CTA a row
  switch (sortn) {
    case 32: route_kernel<1><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 64: route_kernel<2><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 128: route_kernel<4><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 256: route_kernel<8><<<g2, kRouteWarps * 32, 0, s>>>(a); break;
    case 512: route_row_kernel<2><<<(unsigned)rows, kRowThreads, 0, s>>>(a); break;
    case 1024: route_row_kernel<4><<<(unsigned)rows, kRowThreads, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ta
