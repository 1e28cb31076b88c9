// ta_static.cu -- the router without any allocation: its scratch lives in a
// fixed-size array in the library's own device memory.
//
// Some callers cannot allocate device memory at all: code running inside a
// host framework that owns every byte of the GPU (a plugin with a fixed memory
// budget, for instance), or a latency-critical path where a cudaMalloc would
// synchronise the device.  tiered_attn_route_noalloc gives them the tier map
// and the per-row tile lists from Q, K, V and caller-owned output buffers only;
// the block means, pooled logits and masses it needs in between are kept in
// `g_route_scratch` below.  Every GPU that loads the library holds that array
// until the process exits.
#include <cmath>
#include <cstring>
#include <mutex>

#include "ta_common.cuh"
#include "ta_kernels.cuh"

namespace {

constexpr size_t kScratchBytes = TA_ROUTE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_route_scratch on the current device, looked up once per
// device (the array's name in host code is only a host-side stand-in).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

inline size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

void ta_resolve_tier_cost(const ta_params* p, double* cost);

extern "C" ta_status tiered_attn_route_noalloc(const ta_params* p, const void* Q, const void* K,
                                               const void* V, uint8_t* tier_map,
                                               int32_t* row_counts, int32_t* row_lists,
                                               void* stream) {
  if (tiered_attn_workspace_bytes(p) == 0) return TA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !tier_map || !row_counts || !row_lists) return TA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
       reinterpret_cast<uintptr_t>(V)) % 16)
    return TA_ERR_INVALID_ARG;
  const int64_t BH = (int64_t)p->B * p->H;
  const int64_t nQb = (p->N + p->block_q - 1) / p->block_q;
  const int64_t nKb = (p->N + p->block_k - 1) / p->block_k;
  const bool price = p->router == TA_ROUTER_PRICE;
  // scratch sections: status, n_k, qbar, kbar, kbar_b, vbar_b, logits, mass;
  // for the price router also kvar, qvar (block coordinate variances) and
  // spread (the skip tier's error factor)
  constexpr int kSections = 11;
  size_t off[kSections];
  size_t at = 0;
  const size_t sizes[kSections] = {16, (size_t)nKb * 4, (size_t)(BH * nQb * p->d * 8),
                                   (size_t)(BH * nKb * p->d * 8), (size_t)(BH * nKb * p->d * 2),
                                   (size_t)(BH * nKb * p->d * 2), (size_t)(BH * nQb * nKb * 8),
                                   (size_t)(BH * nQb * nKb * 8),
                                   price ? (size_t)(BH * nKb * p->d * 8) : 0,
                                   price ? (size_t)(BH * nQb * p->d * 8) : 0,
                                   price ? (size_t)(BH * nQb * nKb * 8) : 0};
  for (int i = 0; i < kSections; ++i) {
    off[i] = at;
    at = up256(at + sizes[i]);
  }
  if (at > kScratchBytes) return TA_ERR_WORKSPACE;  // problem too large for the fixed scratch

  unsigned char* base = static_cast<unsigned char*>(scratch_on_current_device());
  if (!base) return TA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  ta::PlanArgs a;
  std::memset(&a, 0, sizeof(a));
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
  a.low = TA_LOW_NONE;  // prep: block means (and variances) only, no low-precision copies
  a.R = p->block_q > p->block_k ? p->block_q : p->block_k;
  a.nQb = (int)nQb;
  a.nKb = (int)nKb;
  a.Np = 32 * ((p->N + 31) / 32);
  a.n_tau = p->n_thresholds;
  for (int i = 0; i < 3; ++i) a.tau[i] = i < p->n_thresholds ? p->tau[i] : 0.0;
  a.keep_diag = p->keep_diag_full;
  a.router = p->router;
  a.price = p->price;
  ta_resolve_tier_cost(p, a.cost);
  a.retention = p->retention;
  a.scale = p->softmax_scale > 0.0f ? (double)p->softmax_scale : 1.0 / std::sqrt((double)p->d);
  a.status = reinterpret_cast<int*>(base + off[0]);
  a.n_k = reinterpret_cast<int*>(base + off[1]);
  a.qbar = reinterpret_cast<double*>(base + off[2]);
  a.kbar = reinterpret_cast<double*>(base + off[3]);
  a.kbar_b = reinterpret_cast<__nv_bfloat16*>(base + off[4]);
  a.vbar_b = reinterpret_cast<__nv_bfloat16*>(base + off[5]);
  a.logits = reinterpret_cast<double*>(base + off[6]);
  a.mass = reinterpret_cast<double*>(base + off[7]);
  if (price) {
    a.kvar = reinterpret_cast<double*>(base + off[8]);
    a.qvar = reinterpret_cast<double*>(base + off[9]);
    a.spread = reinterpret_cast<double*>(base + off[10]);
  }
  a.tier_map = tier_map;
  a.row_counts = row_counts;
  a.row_lists = row_lists;

  // the status word is the only scratch that must start from zero; every
  // other section is fully rewritten by the kernels below
  if (cudaMemsetAsync(a.status, 0, 16, s) != cudaSuccess) return TA_ERR_CUDA;
  if (ta::launch_prep(a, s) != cudaSuccess) return TA_ERR_CUDA;
  // the price router chooses among the tiers the low format provides
  a.low = p->low;
  if (ta::launch_route(a, s) != cudaSuccess) return TA_ERR_CUDA;
  return TA_OK;
}
