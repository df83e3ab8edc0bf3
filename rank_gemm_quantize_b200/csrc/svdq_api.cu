// Host side of the C ABI: argument checks, the layer handle, the offline
// preparation pipeline (cuSOLVER float64 SVD between our own kernels), the
// forward's two launches, LoRA attach, export to the canonical layout.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <cudaTypedefs.h>
#include <cusolverDn.h>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "kernels.h"

using namespace svdq;

namespace {

thread_local std::string g_last_error;

svdq_status fail(svdq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

}  // namespace

namespace svdq {
// Lets other translation units of the library report through svdq_last_error.
void set_last_error(const std::string& msg) { g_last_error = msg; }

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tiled tensor map: inner dimension contiguous, rows row_bytes apart.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace svdq

namespace {

#define CUDA_TRY(expr)                                                                              \
  do {                                                                                              \
    cudaError_t e__ = (expr);                                                                       \
    if (e__ != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e__)); \
  } while (0)

inline int round_up(int v, int m) { return (v + m - 1) / m * m; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Weight-side padding: every GEMM tile width divides it, so per-tile scale
// copies never leave the buffers.
constexpr int kNPad = 256;

// Small cache of tensor maps keyed by (device pointer, rows): encoding a map
// costs microseconds of host time, and callers usually cycle through a few
// buffers.
template <int N>
struct MapCache {
  struct Entry {
    const void* key = nullptr;
    int rows = -1;
    CUtensorMap a{}, b{}, c{}, d{};
    const void* dkey = nullptr;  // the buffer map d was made for (built on first use)
  };
  Entry e[N];
  int next = 0;
  Entry* find(const void* key, int rows) {
    for (auto& x : e)
      if (x.key == key && x.rows == rows) return &x;
    return nullptr;
  }
  Entry* insert(const void* key, int rows) {
    Entry* x = &e[next];
    next = (next + 1) % N;
    x->key = key;
    x->rows = rows;
    return x;
  }
  void clear() {
    for (auto& x : e) x = Entry{};
  }
};

struct WsLayout {
  int M_pad;
  int split;      // activation-kernel K shares per 128-row block
  size_t codes, scales, T, Tpart, total;
};

}  // namespace

struct svdq_layer {
  int device = 0;
  int sms = 148;  // SM count of the device, read at preparation
  int k1_per_sm = 1;  // resident activation-kernel CTAs per SM (format, rank padding), read at prepare / attach
  svdq_config cfg{};
  int K = 0, N = 0, N_pad = 0;
  int rank = 0, RP = 0;  // branch rank (base + attached adapters) and its padding to a multiple of 32 (0 when empty)
  int fmt = 0;
  float g_x = 1.f, g_w = 1.f, gxgw = 1.f, t_scale = 1.f, denom = 6.f;
  float* s = nullptr;
  float* inv_s = nullptr;
  // The branch as blocks of columns: the base factors (rank base_rank) and one
  // block per occupied adapter slot, each as F [K, r] and G [r, N] (bf16).
  int base_rank = 0;
  __nv_bfloat16* base_F = nullptr;  // L1 [K, base_rank]
  __nv_bfloat16* base_G = nullptr;  // L2 [base_rank, N]
  struct Adapter {
    int rank = 0;  // 0: slot free
    __nv_bfloat16* F = nullptr;  // bf16(diag(s) A) [K, rank]
    __nv_bfloat16* G = nullptr;  // bf16(scale B) [rank, N]
  } adapters[kMaxAdapters];
  int col_start[kMaxAdapters + 1] = {};  // slot s owns branch columns [col_start[s], col_start[s+1])
  // ... assembled in slot order into the layouts the kernels read:
  __nv_bfloat16* L1T = nullptr;    // [RP, K]  canonical L1'^T
  __nv_bfloat16* L1sTh = nullptr;  // [RP, K]  bf16 hi of fp32(inv_s[k] L1'[k, j])
  __nv_bfloat16* L1sTl = nullptr;  // [RP, K]  bf16 lo of the same
  __nv_bfloat16* L2T = nullptr;    // [N_pad, RP] canonical L2'^T
  __nv_bfloat16* bias = nullptr; // [N_pad], zero beyond N
  uint8_t* wcodes = nullptr;     // INT4 [N_pad, K] E4M3 bytes; NVFP4 [N_pad, K/2]
  void* wscales = nullptr;       // INT4 float [K/64][N_pad]; NVFP4 atoms [N_pad/128][K/64][512]
  int* status = nullptr;         // device status word
  int* k1_counters = nullptr;    // activation-kernel arrival counters per 128-row block (zero between launches)
  CUtensorMap map_b{}, map_l2{}, map_l1h{}, map_l1l{}, map_sfb{};
  // as the down layer of a fused MLP block: L1s^T hi / lo with 16-row boxes
  CUtensorMap map_l1h_half{}, map_l1l_half{};
  bool mlp_maps_ready = false;
  MapCache<8> ws_maps;  // (workspace, M) -> activation codes map (a), T map (b)
  MapCache<8> x_maps;   // (X, M) -> X map (a)
  MapCache<8> y_maps;   // (Y, M) -> Y map (a), NVFP4 only
};

namespace {

WsLayout ws_layout(const svdq_layer* h, int M) {
  WsLayout w{};
  w.M_pad = round_up(M, 128);
  const size_t cbytes = h->fmt == SVDQ_INT4_G64 ? static_cast<size_t>(w.M_pad) * h->K
                                                : static_cast<size_t>(w.M_pad) * (h->K / 2);
  const size_t sbytes = h->fmt == SVDQ_INT4_G64 ? static_cast<size_t>(h->K / 64) * w.M_pad * 4
                                                : static_cast<size_t>(w.M_pad / 128) * (h->K / 64) * 512;
  w.codes = 0;
  w.scales = align256(cbytes);
  w.split = act_quant_split(w.M_pad, h->K, h->k1_per_sm, h->sms);
  w.T = w.scales + align256(sbytes);
  w.Tpart = w.T + align256(static_cast<size_t>(w.M_pad) * h->RP * 2);
  const size_t part = w.split > 1 && h->RP > 0 ? static_cast<size_t>(w.split) * w.M_pad * h->RP * 4 : 0;
  w.total = w.Tpart + align256(part);
  return w;
}

svdq_status check_device() {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  int major = 0, minor = 0;
  CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0) return fail(SVDQ_ERR_UNSUPPORTED, "svdq needs an sm_100 (B200-class) device");
  return SVDQ_OK;
}

svdq_status check_cfg(const svdq_config* cfg) {
  if (!cfg) return fail(SVDQ_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->K <= 0 || cfg->K % 128) return fail(SVDQ_ERR_INVALID_ARG, "K must be a positive multiple of 128");
  if (cfg->N <= 0 || cfg->N % 16) return fail(SVDQ_ERR_INVALID_ARG, "N must be a positive multiple of 16");
  if (cfg->rank < 0 || cfg->rank > 256) return fail(SVDQ_ERR_INVALID_ARG, "rank must be in [0, 256]");
  if (cfg->rank > std::min(cfg->K, cfg->N)) return fail(SVDQ_ERR_INVALID_ARG, "rank exceeds min(K, N)");
  if (!(cfg->alpha >= 0.f && cfg->alpha <= 1.f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (!(cfg->s_min > 0.f) || !std::isfinite(cfg->s_min)) return fail(SVDQ_ERR_INVALID_ARG, "s_min must be > 0");
  if (cfg->fmt != SVDQ_INT4_G64 && cfg->fmt != SVDQ_NVFP4_G16) return fail(SVDQ_ERR_INVALID_ARG, "unknown format");
  if (cfg->flags & ~static_cast<unsigned>(SVDQ_NO_SMOOTHING)) return fail(SVDQ_ERR_INVALID_ARG, "unknown flags");
  return SVDQ_OK;
}

// Test hook (svdq_debug_fail_allocation): the library's device allocation
// with this index (counting from the hook's call) fails as if the device were
// out of memory; -1 disables it.
std::atomic<long long> g_fail_alloc_at{-1};

bool injected_alloc_failure() {
  long long v = g_fail_alloc_at.load(std::memory_order_relaxed);
  while (v >= 0) {
    if (g_fail_alloc_at.compare_exchange_weak(v, v - 1, std::memory_order_relaxed)) return v == 0;
  }
  return false;
}

template <class T>
svdq_status dalloc(T** p, size_t bytes) {
  *p = nullptr;
  if (injected_alloc_failure()) return fail(SVDQ_ERR_OOM, "device allocation failed (injected by the test hook)");
  if (cudaMalloc(reinterpret_cast<void**>(p), std::max<size_t>(bytes, 256)) != cudaSuccess) {
    cudaGetLastError();
    return fail(SVDQ_ERR_OOM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed");
  }
  return SVDQ_OK;
}

void free_layer(svdq_layer* h) {
  if (!h) return;
  cudaFree(h->s);
  cudaFree(h->inv_s);
  cudaFree(h->base_F);
  cudaFree(h->base_G);
  for (auto& a : h->adapters) {
    cudaFree(a.F);
    cudaFree(a.G);
  }
  cudaFree(h->L1T);
  cudaFree(h->L1sTh);
  cudaFree(h->L1sTl);
  cudaFree(h->L2T);
  cudaFree(h->bias);
  cudaFree(h->wcodes);
  cudaFree(h->wscales);
  cudaFree(h->status);
  cudaFree(h->k1_counters);
  delete h;
}

// NVFP4 scale-factor atoms (512 bytes each) as a uint32 [atoms, 128] tensor,
// loaded four atoms (the four 64-wide k-blocks of a 256-deep k-tile) at a time.
bool make_sf_map(CUtensorMap* m, const void* base, uint64_t atoms) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, base, 128, atoms, 512, 128, 4, CU_TENSOR_MAP_SWIZZLE_NONE);
}

svdq_status build_static_maps(svdq_layer* h) {
  const bool i4 = h->fmt == SVDQ_INT4_G64;
  const uint64_t row = i4 ? h->K : h->K / 2;
  if (!make_map(&h->map_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->wcodes, row, h->N_pad, row, 128, kWeightBoxRows,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (weight codes) failed");
  h->map_sfb = CUtensorMap{};
  if (!i4 && !make_sf_map(&h->map_sfb, h->wscales, static_cast<uint64_t>(h->N_pad / 128) * (h->K / 64)))
    return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (weight scale factors) failed");
  h->map_l2 = CUtensorMap{};
  h->map_l1h = CUtensorMap{};
  h->map_l1l = CUtensorMap{};
  if (h->RP > 0) {
    if (!make_map(&h->map_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->L2T, h->RP, h->N_pad,
                  static_cast<uint64_t>(h->RP) * 2, 32, kWeightBoxRows, CU_TENSOR_MAP_SWIZZLE_64B))
      return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (L2) failed");
    if (!make_map(&h->map_l1h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->L1sTh, h->K, h->RP, static_cast<uint64_t>(h->K) * 2,
                  64, h->RP, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&h->map_l1l, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->L1sTl, h->K, h->RP, static_cast<uint64_t>(h->K) * 2,
                  64, h->RP, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (L1) failed");
  }
  h->ws_maps.clear();
  h->x_maps.clear();
  h->y_maps.clear();
  h->mlp_maps_ready = false;
  return SVDQ_OK;
}

// Host part of eq. 2 (float64, one rounding to float32), plus the NVFP4 static
// activation tensor scale.
void smoothing_host(const std::vector<float>& a, const std::vector<float>& w, float alpha, float s_min, bool smooth,
                    std::vector<float>& s, std::vector<float>& inv_s) {
  const size_t K = a.size();
  s.resize(K);
  inv_s.resize(K);
  for (size_t k = 0; k < K; ++k) {
    double sk;
    if (!smooth) {  // the no-smoothing ablation: s = 1 for every channel
      s[k] = 1.0f;
      inv_s[k] = 1.0f;
      continue;
    }
    if (a[k] == 0.f || w[k] == 0.f) {
      sk = 1.0;
    } else if (alpha == 0.5f) {
      sk = std::sqrt(static_cast<double>(a[k])) / std::sqrt(static_cast<double>(w[k]));
    } else {
      sk = std::pow(static_cast<double>(a[k]), static_cast<double>(alpha)) /
           std::pow(static_cast<double>(w[k]), 1.0 - static_cast<double>(alpha));
    }
    const float f = std::max(static_cast<float>(sk), s_min);  // s >= s_min for every channel
    s[k] = f;
    inv_s[k] = 1.0f / f;
  }
}

float nvfp4_tensor_scale_host(float amax) {
  if (amax == 0.f) return 1.0f;
  volatile float d = 2688.0f;
  return amax / d;
}

// (Re)builds the kernel layouts of the branch from its blocks (the base
// factors, then the occupied adapter slots in slot order) into new buffers,
// and swaps them in only when everything succeeded: on failure the layer is
// unchanged. Synchronizes `st` before freeing the previous buffers.
svdq_status assemble_branch(svdq_layer* h, cudaStream_t st) {
  int cs[kMaxAdapters + 1];
  cs[0] = h->base_rank;
  for (int a = 0; a < kMaxAdapters; ++a) cs[a + 1] = cs[a] + h->adapters[a].rank;
  const int rank = cs[kMaxAdapters];
  if (rank > 256) return fail(SVDQ_ERR_INVALID_ARG, "branch rank (base + adapters) exceeds 256");
  const int RP = round_up(rank, 32);
  __nv_bfloat16 *L1T = nullptr, *L1sTh = nullptr, *L1sTl = nullptr, *L2T = nullptr;
  auto drop = [&] {
    cudaFree(L1T);
    cudaFree(L1sTh);
    cudaFree(L1sTl);
    cudaFree(L2T);
  };
  if (RP > 0) {
    const size_t l1 = static_cast<size_t>(RP) * h->K * 2, l2 = static_cast<size_t>(h->N_pad) * RP * 2;
    svdq_status e;
    if ((e = dalloc(&L1T, l1)) || (e = dalloc(&L1sTh, l1)) || (e = dalloc(&L1sTl, l1)) || (e = dalloc(&L2T, l2)))
      return drop(), e;
    cudaError_t ce = cudaMemsetAsync(L1T, 0, l1, st);
    if (ce == cudaSuccess) ce = cudaMemsetAsync(L1sTh, 0, l1, st);
    if (ce == cudaSuccess) ce = cudaMemsetAsync(L1sTl, 0, l1, st);
    if (ce == cudaSuccess) ce = cudaMemsetAsync(L2T, 0, l2, st);
    if (ce == cudaSuccess && h->base_rank > 0)
      ce = launch_assemble_block(h->base_F, h->base_G, h->base_rank, 0, h->K, h->N, RP, h->inv_s, L1T, L1sTh, L1sTl,
                                 L2T, st);
    for (int a = 0; a < kMaxAdapters && ce == cudaSuccess; ++a)
      if (h->adapters[a].rank > 0)
        ce = launch_assemble_block(h->adapters[a].F, h->adapters[a].G, h->adapters[a].rank, cs[a], h->K, h->N, RP,
                                   h->inv_s, L1T, L1sTh, L1sTl, L2T, st);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
    if (ce != cudaSuccess) return drop(), fail(SVDQ_ERR_CUDA, std::string("branch assembly: ") + cudaGetErrorString(ce));
  } else {
    cudaError_t ce = cudaStreamSynchronize(st);  // earlier work on the old buffers is done before they go
    if (ce != cudaSuccess) return fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
  }
  cudaFree(h->L1T);
  cudaFree(h->L1sTh);
  cudaFree(h->L1sTl);
  cudaFree(h->L2T);
  h->L1T = L1T;
  h->L1sTh = L1sTh;
  h->L1sTl = L1sTl;
  h->L2T = L2T;
  h->rank = rank;
  h->RP = RP;
  for (int a = 0; a <= kMaxAdapters; ++a) h->col_start[a] = cs[a];
  h->k1_per_sm = act_quant_resident(h->fmt, h->RP);
  return build_static_maps(h);
}

// Steps shared by both prepare entry points once L1 [K, rank] and L2 [rank, N]
// (bf16, device) exist: residual, quantization, branch layout.
svdq_status finish_prepare(svdq_layer* h, const float* W_hat, const __nv_bfloat16* L1, const __nv_bfloat16* L2,
                           cudaStream_t st) {
  const int K = h->K, N = h->N;
  float* R = nullptr;
  svdq_status e = dalloc(&R, static_cast<size_t>(K) * N * 4);
  if (e) return e;
  auto cleanup = [&] { cudaFree(R); };
  if (launch_residual(W_hat, L1, L2, K, N, h->base_rank, R, st) != cudaSuccess) {
    cleanup();
    return fail(SVDQ_ERR_CUDA, "residual kernel launch failed");
  }
  if (h->fmt == SVDQ_INT4_G64) {
    if ((e = dalloc(&h->wcodes, static_cast<size_t>(h->N_pad) * K))) return cleanup(), e;
    if ((e = dalloc(reinterpret_cast<float**>(&h->wscales), static_cast<size_t>(K / 64) * h->N_pad * 4))) return cleanup(), e;
    cudaMemsetAsync(h->wcodes, 0, static_cast<size_t>(h->N_pad) * K, st);
    cudaMemsetAsync(h->wscales, 0, static_cast<size_t>(K / 64) * h->N_pad * 4, st);
    if (launch_quant_weight_int4(R, K, N, h->N_pad, h->wcodes, static_cast<float*>(h->wscales), st) != cudaSuccess)
      return cleanup(), fail(SVDQ_ERR_CUDA, "weight quantization launch failed");
  } else {
    unsigned int* amax = nullptr;
    float* gw_dev = nullptr;
    if ((e = dalloc(&h->wcodes, static_cast<size_t>(h->N_pad) * K / 2))) return cleanup(), e;
    if ((e = dalloc(reinterpret_cast<uint8_t**>(&h->wscales), static_cast<size_t>(h->N_pad / 128) * (K / 64) * 512)))
      return cleanup(), e;
    if ((e = dalloc(&amax, 16))) return cleanup(), e;
    gw_dev = reinterpret_cast<float*>(amax) + 1;
    cudaMemsetAsync(h->wcodes, 0, static_cast<size_t>(h->N_pad) * K / 2, st);
    cudaMemsetAsync(h->wscales, 0, static_cast<size_t>(h->N_pad / 128) * (K / 64) * 512, st);
    cudaMemsetAsync(amax, 0, 16, st);
    if (launch_absmax_all(R, static_cast<size_t>(K) * N, amax, st) != cudaSuccess ||
        launch_quant_weight_nvfp4(R, K, N, h->N_pad, amax, h->wcodes, static_cast<uint8_t*>(h->wscales), gw_dev, st) !=
            cudaSuccess) {
      cudaFree(amax);
      return cleanup(), fail(SVDQ_ERR_CUDA, "weight quantization launch failed");
    }
    float gw = 1.f;
    cudaError_t ce = cudaMemcpyAsync(&gw, gw_dev, 4, cudaMemcpyDeviceToHost, st);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
    cudaFree(amax);
    if (ce != cudaSuccess) return cleanup(), fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
    h->g_w = gw;
  }
  // the base block of the branch: the layer keeps its own copy of L1, L2
  if (h->base_rank > 0) {
    const size_t f = static_cast<size_t>(K) * h->base_rank * 2, g = static_cast<size_t>(h->base_rank) * N * 2;
    if ((e = dalloc(&h->base_F, f)) || (e = dalloc(&h->base_G, g))) return cleanup(), e;
    cudaError_t ce = cudaMemcpyAsync(h->base_F, L1, f, cudaMemcpyDeviceToDevice, st);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(h->base_G, L2, g, cudaMemcpyDeviceToDevice, st);
    if (ce != cudaSuccess) return cleanup(), fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
  }
  cudaError_t ce = cudaStreamSynchronize(st);
  cleanup();
  if (ce != cudaSuccess) return fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
  if (h->fmt == SVDQ_NVFP4_G16) {
    h->gxgw = h->g_x * h->g_w;
    h->t_scale = 1.0f / h->gxgw;
  } else {
    h->gxgw = 1.f;
    h->t_scale = 1.f;
  }
  return assemble_branch(h, st);
}

// Steps 1 (statistics, eq. 2) and the migration of eq. 1.
svdq_status start_prepare(const svdq_config* cfg, const void* W, const void* bias, const float* act_absmax,
                          cudaStream_t st, svdq_layer** out_h, float** W_hat_out) {
  svdq_status e;
  // arguments first: a bad call is refused before the device is touched
  if ((e = check_cfg(cfg))) return e;
  if (!W || !act_absmax) return fail(SVDQ_ERR_INVALID_ARG, "W and act_absmax must not be NULL");
  if (!aligned16(W) || (bias && !aligned16(bias)) || !aligned16(act_absmax))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if ((e = check_device())) return e;
  svdq_layer* h = new svdq_layer();
  cudaGetDevice(&h->device);
  if (cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess || h->sms < 1) {
    cudaGetLastError();
    h->sms = 148;
  }
  h->cfg = *cfg;
  h->K = cfg->K;
  h->N = cfg->N;
  h->N_pad = round_up(cfg->N, kNPad);
  h->base_rank = cfg->rank;
  h->fmt = cfg->fmt;
  const int K = h->K, N = h->N;
  auto bail = [&](svdq_status s) {
    free_layer(h);
    return s;
  };
  if ((e = dalloc(&h->s, K * 4)) || (e = dalloc(&h->inv_s, K * 4)) || (e = dalloc(&h->bias, h->N_pad * 2)) ||
      (e = dalloc(&h->status, 16)) || (e = dalloc(&h->k1_counters, kMaxRowBlocks * sizeof(int))))
    return bail(e);
  cudaMemsetAsync(h->status, 0, 16, st);
  cudaMemsetAsync(h->k1_counters, 0, kMaxRowBlocks * sizeof(int), st);
  cudaMemsetAsync(h->bias, 0, h->N_pad * 2, st);  // padded with zeros to the weight padding
  if (bias) cudaMemcpyAsync(h->bias, bias, N * 2, cudaMemcpyDeviceToDevice, st);

  float* wstat = nullptr;
  if ((e = dalloc(&wstat, K * 4))) return bail(e);
  if (launch_absmax_rows(static_cast<const __nv_bfloat16*>(W), K, N, wstat, st) != cudaSuccess) {
    cudaFree(wstat);
    return bail(fail(SVDQ_ERR_CUDA, "absmax kernel launch failed"));
  }
  std::vector<float> a(K), w(K), s, inv_s;
  cudaError_t ce = cudaMemcpyAsync(a.data(), act_absmax, K * 4, cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(w.data(), wstat, K * 4, cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  cudaFree(wstat);
  if (ce != cudaSuccess) return bail(fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce)));
  for (int k = 0; k < K; ++k)
    if (!(a[k] >= 0.f) || !std::isfinite(a[k])) return bail(fail(SVDQ_ERR_INVALID_ARG, "act_absmax must be finite and >= 0"));
  smoothing_host(a, w, cfg->alpha, cfg->s_min, (cfg->flags & SVDQ_NO_SMOOTHING) == 0, s, inv_s);
  if (cfg->fmt == SVDQ_NVFP4_G16) {
    float amax_x = 0.f;
    for (int k = 0; k < K; ++k) {
      volatile float prod = a[k] * inv_s[k];
      amax_x = std::max(amax_x, static_cast<float>(prod));
    }
    h->g_x = nvfp4_tensor_scale_host(amax_x);
    volatile float six = 6.0f;
    h->denom = six * h->g_x;
  }
  ce = cudaMemcpyAsync(h->s, s.data(), K * 4, cudaMemcpyHostToDevice, st);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(h->inv_s, inv_s.data(), K * 4, cudaMemcpyHostToDevice, st);
  if (ce != cudaSuccess) return bail(fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce)));
  float* W_hat = nullptr;
  if ((e = dalloc(&W_hat, static_cast<size_t>(K) * N * 4))) return bail(e);
  if (launch_migrate(static_cast<const __nv_bfloat16*>(W), h->s, K, N, W_hat, st) != cudaSuccess) {
    cudaFree(W_hat);
    return bail(fail(SVDQ_ERR_CUDA, "migrate kernel launch failed"));
  }
  ce = cudaStreamSynchronize(st);
  if (ce != cudaSuccess) {
    cudaFree(W_hat);
    return bail(fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce)));
  }
  *out_h = h;
  *W_hat_out = W_hat;
  return SVDQ_OK;
}

// Truncated SVD of W_hat with cuSOLVER (float64 gesvd on whichever
// orientation has m >= n), then L1, L2 in bf16.
svdq_status svd_factors(svdq_layer* h, const float* W_hat, __nv_bfloat16* L1, __nv_bfloat16* L2, cudaStream_t st) {
  const int K = h->K, N = h->N;
  const bool wt = N >= K;  // SVD of W_hat^T (N x K) when N >= K, else of W_hat (K x N)
  const int m = wt ? N : K, n = wt ? K : N;
  double *A = nullptr, *S = nullptr, *U = nullptr, *VT = nullptr, *work = nullptr, *rwork = nullptr;
  int* info = nullptr;
  svdq_status e = SVDQ_OK;
  cusolverDnHandle_t sh = nullptr;
  auto cleanup = [&] {
    cudaFree(A);
    cudaFree(S);
    cudaFree(U);
    cudaFree(VT);
    cudaFree(work);
    cudaFree(rwork);
    cudaFree(info);
    if (sh) cusolverDnDestroy(sh);
  };
  if ((e = dalloc(&A, static_cast<size_t>(m) * n * 8)) || (e = dalloc(&S, static_cast<size_t>(n) * 8)) ||
      (e = dalloc(&U, static_cast<size_t>(m) * n * 8)) || (e = dalloc(&VT, static_cast<size_t>(n) * n * 8)) ||
      (e = dalloc(&rwork, static_cast<size_t>(n) * 8)) || (e = dalloc(&info, 16)))
    return cleanup(), e;
  if (launch_to_f64_colmajor(W_hat, K, N, !wt, A, st) != cudaSuccess)
    return cleanup(), fail(SVDQ_ERR_CUDA, "layout kernel launch failed");
  if (cusolverDnCreate(&sh) != CUSOLVER_STATUS_SUCCESS) return cleanup(), fail(SVDQ_ERR_CUDA, "cusolverDnCreate failed");
  cusolverDnSetStream(sh, st);
  int lwork = 0;
  if (cusolverDnDgesvd_bufferSize(sh, m, n, &lwork) != CUSOLVER_STATUS_SUCCESS)
    return cleanup(), fail(SVDQ_ERR_CUDA, "gesvd_bufferSize failed");
  if ((e = dalloc(&work, static_cast<size_t>(lwork) * 8))) return cleanup(), e;
  signed char jobu = 'S', jobvt = 'S';
  if (cusolverDnDgesvd(sh, jobu, jobvt, m, n, A, m, S, U, m, VT, n, work, lwork, rwork, info) !=
      CUSOLVER_STATUS_SUCCESS)
    return cleanup(), fail(SVDQ_ERR_CUDA, "gesvd failed to launch");
  int hinfo = 0;
  cudaError_t ce = cudaMemcpyAsync(&hinfo, info, 4, cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  if (ce != cudaSuccess) return cleanup(), fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
  if (hinfo != 0) return cleanup(), fail(SVDQ_ERR_NUMERIC, "gesvd did not converge (info=" + std::to_string(hinfo) + ")");
  if (launch_factors_from_svd(U, S, VT, K, N, h->base_rank, wt, m, n, L1, L2, st) != cudaSuccess)
    return cleanup(), fail(SVDQ_ERR_CUDA, "factor kernel launch failed");
  ce = cudaStreamSynchronize(st);
  cleanup();
  if (ce != cudaSuccess) return fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
  return SVDQ_OK;
}

svdq_status launch_k1(svdq_layer* h, const void* X, int M, uint8_t* codes, void* scales, __nv_bfloat16* T,
                      float* Tpart, const WsLayout& w, const uint32_t* row_mask, cudaStream_t st,
                      __nv_bfloat16* T_lo = nullptr) {
  if (w.M_pad / 128 > kMaxRowBlocks) return fail(SVDQ_ERR_INVALID_ARG, "M exceeds the supported row count");
  ActQuantParams p{};
  p.split = w.split;
  p.Tpart = Tpart;
  p.counters = h->k1_counters;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.M = M;
  p.K = h->K;
  p.M_pad = round_up(M, 128);
  p.inv_s = h->inv_s;
  p.codes = codes;
  p.scales = scales;
  p.T = T;
  p.T_lo = T_lo;
  p.g_x = h->g_x;
  p.denom = h->denom;
  p.t_scale = h->t_scale;
  p.status = h->status;
  p.row_mask = row_mask;
  for (int a = 0; a <= kMaxAdapters; ++a) p.col_start[a] = h->col_start[a];
  ActQuantMaps maps;
  auto* xe = h->x_maps.find(X, M);
  if (!xe) {
    xe = h->x_maps.insert(X, M);
    if (!make_map(&xe->a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, h->K, M, static_cast<uint64_t>(h->K) * 2, 64,
                  act_quant_box_rows(), CU_TENSOR_MAP_SWIZZLE_128B)) {
      xe->key = nullptr;
      return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (X) failed");
    }
  }
  maps.x = xe->a;
  maps.l1h = h->map_l1h;
  maps.l1l = h->map_l1l;
  cudaError_t e = launch_act_quant(p, maps, h->fmt, h->RP, st);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("activation kernel: ") + cudaGetErrorString(e));
  return SVDQ_OK;
}

svdq_status check_layer(svdq_layer* h) {
  if (!h) return fail(SVDQ_ERR_INVALID_ARG, "layer is NULL");
  return SVDQ_OK;
}

// Calls that launch kernels on a layer's buffers must run with the layer's
// device current: its weights, tensor maps and scratch live there.
svdq_status check_layer_device(svdq_layer* h) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev != h->device)
    return fail(SVDQ_ERR_INVALID_ARG, "the current device (" + std::to_string(dev) + ") is not the layer's device (" +
                                          std::to_string(h->device) + ")");
  return SVDQ_OK;
}

}  // namespace

extern "C" {

const char* svdq_last_error(void) { return g_last_error.c_str(); }

svdq_status svdq_calibrate_absmax(const void* X, int M, int K, float* absmax_inout, void* stream) {
  if (!X || !absmax_inout || M < 1 || K < 1) return fail(SVDQ_ERR_INVALID_ARG, "bad calibration arguments");
  if (!aligned16(X) || !aligned16(absmax_inout)) return fail(SVDQ_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (launch_absmax_cols(static_cast<const __nv_bfloat16*>(X), M, K, absmax_inout, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return fail(SVDQ_ERR_CUDA, "calibration kernel launch failed");
  return SVDQ_OK;
}

svdq_status svdq_prepare_weights(const svdq_config* cfg, const void* W, const void* bias, const float* act_absmax,
                                 void* stream, svdq_layer_t* out) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  svdq_layer* h = nullptr;
  float* W_hat = nullptr;
  svdq_status e = start_prepare(cfg, W, bias, act_absmax, st, &h, &W_hat);
  if (e) return e;
  __nv_bfloat16 *L1 = nullptr, *L2 = nullptr;
  // rank 0 (smoothing only, no branch) needs no decomposition
  if (h->base_rank > 0 && ((e = dalloc(&L1, static_cast<size_t>(h->K) * h->base_rank * 2)) ||
                           (e = dalloc(&L2, static_cast<size_t>(h->base_rank) * h->N * 2)) ||
                           (e = svd_factors(h, W_hat, L1, L2, st))))
    ;
  if (e == SVDQ_OK) e = finish_prepare(h, W_hat, L1, L2, st);
  if (e) {
    cudaFree(L1);
    cudaFree(L2);
    cudaFree(W_hat);
    free_layer(h);
    return e;
  }
  cudaFree(L1);
  cudaFree(L2);
  cudaFree(W_hat);
  *out = h;
  return SVDQ_OK;
}

svdq_status svdq_prepare_weights_with_factors(const svdq_config* cfg, const void* W, const void* bias,
                                              const float* act_absmax, const void* L1, const void* L2, void* stream,
                                              svdq_layer_t* out) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (cfg && cfg->rank > 0 && (!L1 || !L2)) return fail(SVDQ_ERR_INVALID_ARG, "L1 and L2 must not be NULL");
  if ((L1 && !aligned16(L1)) || (L2 && !aligned16(L2)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  svdq_layer* h = nullptr;
  float* W_hat = nullptr;
  svdq_status e = start_prepare(cfg, W, bias, act_absmax, st, &h, &W_hat);
  if (e) return e;
  e = finish_prepare(h, W_hat, static_cast<const __nv_bfloat16*>(L1), static_cast<const __nv_bfloat16*>(L2), st);
  cudaFree(W_hat);
  if (e) {
    free_layer(h);
    return e;
  }
  *out = h;
  return SVDQ_OK;
}

svdq_status svdq_workspace_size(svdq_layer_t h, int M, size_t* bytes) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (!bytes || M < 1) return fail(SVDQ_ERR_INVALID_ARG, "bad workspace query");
  *bytes = ws_layout(h, M).total;
  return SVDQ_OK;
}

}  // extern "C"

namespace {

// The GEMM of a forward on activations already in the layer's layouts
// (codes, scales, T for M rows). With mlp set (NVFP4 only) the GEMM is the up
// layer of an MLP block: its epilogue writes the down layer's activations
// instead of Y.
svdq_status gemm_stage(svdq_layer* h, int M, void* Y, uint8_t* codes, void* scales, __nv_bfloat16* T,
                       __nv_bfloat16* T_lo, const MlpDownParams* mlp, const GemmMaps* mlp_maps, cudaStream_t st) {
  const int M_pad = round_up(M, 128);
  auto* we = h->ws_maps.find(codes, M);
  if (!we) {
    we = h->ws_maps.insert(codes, M);
    const bool i4 = h->fmt == SVDQ_INT4_G64;
    const uint64_t row = i4 ? h->K : h->K / 2;
    we->b = CUtensorMap{};
    we->c = CUtensorMap{};
    we->d = CUtensorMap{};
    we->dkey = nullptr;
    if (!make_map(&we->a, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, row, M_pad, row, 128, kActBoxRows,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        (!i4 && !make_sf_map(&we->c, scales, static_cast<uint64_t>(M_pad / 128) * (h->K / 64))) ||
        (h->RP > 0 && !make_map(&we->b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, h->RP, M_pad,
                                static_cast<uint64_t>(h->RP) * 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))) {
      we->key = nullptr;
      return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (activations) failed");
    }
  }
  if (h->RP > 0 && T_lo && we->dkey != T_lo) {  // the MLP block's T low part
    if (!make_map(&we->d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T_lo, h->RP, M_pad, static_cast<uint64_t>(h->RP) * 2, 32,
                  128, CU_TENSOR_MAP_SWIZZLE_64B)) {
      we->key = nullptr;
      return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (T low part) failed");
    }
    we->dkey = T_lo;
  }
  GemmParams p{};
  p.M = M;
  p.N = h->N;
  p.K = h->K;
  p.RP = h->RP;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.bias = h->bias;
  p.sa = scales;
  p.sb = h->wscales;
  p.M_pad = M_pad;
  p.N_pad = h->N_pad;
  p.out_scale = h->gxgw;
  p.status = h->status;
  GemmMaps maps = mlp_maps ? *mlp_maps : GemmMaps{};
  maps.a = we->a;
  maps.b = h->map_b;
  maps.t = we->b;
  maps.l2 = h->map_l2;
  maps.sfa = we->c;
  maps.sfb = h->map_sfb;
  maps.t_lo = we->d;
  if (h->fmt == SVDQ_NVFP4_G16 && !mlp) {
    auto* ye = h->y_maps.find(Y, M);
    if (!ye) {
      ye = h->y_maps.insert(Y, M);
      if (!make_map(&ye->a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, h->N, M, static_cast<uint64_t>(h->N) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B)) {
        ye->key = nullptr;
        return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (Y) failed");
      }
    }
    maps.y = ye->a;
  }
  cudaError_t ce;
  if (mlp)
    ce = launch_gemm_nvfp4_mlp(p, *mlp, maps, st);
  else
    ce = h->fmt == SVDQ_INT4_G64 ? launch_gemm_int4(p, maps, st) : launch_gemm_nvfp4(p, maps, st);
  if (ce != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("GEMM kernel: ") + cudaGetErrorString(ce));
  return SVDQ_OK;
}

svdq_status forward_impl(svdq_layer* h, const void* X, int M, void* Y, void* workspace, size_t ws_bytes,
                         const uint32_t* row_mask, void* stream, void* const* events) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (!X || !Y || !workspace || M < 1) return fail(SVDQ_ERR_INVALID_ARG, "NULL pointer or M < 1");
  if (!aligned16(X) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(SVDQ_ERR_INVALID_ARG, "X/Y must be 16-byte and the workspace 256-byte aligned");
  if (row_mask && (reinterpret_cast<uintptr_t>(row_mask) & 3))
    return fail(SVDQ_ERR_INVALID_ARG, "row_mask must be 4-byte aligned");
  const WsLayout w = ws_layout(h, M);
  if (ws_bytes < w.total) return fail(SVDQ_ERR_INVALID_ARG, "workspace too small");
  if (svdq_status e = check_layer_device(h)) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint8_t* codes = base + w.codes;
  void* scales = base + w.scales;
  __nv_bfloat16* T = reinterpret_cast<__nv_bfloat16*>(base + w.T);
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[0]), st));
  float* Tpart = reinterpret_cast<float*>(base + w.Tpart);
  svdq_status e = launch_k1(h, X, M, codes, scales, T, Tpart, w, row_mask, st);
  if (e) return e;
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[1]), st));
  if ((e = gemm_stage(h, M, Y, codes, scales, T, nullptr, nullptr, nullptr, st))) return e;
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[2]), st));
  return SVDQ_OK;
}

// Workspace of an MLP block forward: the up layer's forward workspace, the
// down layer's activation codes, scales and T, and the T partials.
struct MlpLayout {
  WsLayout up, down;
  size_t down_off, tpart_off, tlo_off, total;
  int tiles, n_blocks, pairs, slots;
};

MlpLayout mlp_layout(const svdq_layer* up, const svdq_layer* down, int M) {
  MlpLayout l{};
  l.up = ws_layout(up, M);
  l.down = ws_layout(down, M);
  l.down_off = align256(l.up.total);
  l.tpart_off = l.down_off + align256(l.down.Tpart);  // the down layer's codes, scales and T only
  l.n_blocks = up->N_pad / 256;
  l.tiles = ((l.up.M_pad + 255) / 256) * l.n_blocks;
  l.pairs = nvfp4_pairs(l.tiles);
  l.slots = nvfp4_mlp_slots(l.tiles, l.n_blocks, l.pairs);
  const size_t tpart = static_cast<size_t>((l.up.M_pad + 255) / 256) * l.slots * 256 * kMlpDownRP * 4;
  l.tlo_off = l.tpart_off + align256(tpart);  // the up layer's T low part
  l.total = l.tlo_off + align256(static_cast<size_t>(l.up.M_pad) * up->RP * 2);
  return l;
}

svdq_status check_mlp(svdq_layer* up, svdq_layer* down) {
  if (!up || !down) return fail(SVDQ_ERR_INVALID_ARG, "layer is NULL");
  if (up->fmt != SVDQ_NVFP4_G16 || down->fmt != SVDQ_NVFP4_G16)
    return fail(SVDQ_ERR_UNSUPPORTED, "the fused MLP block needs two NVFP4 layers");
  if (up->N != down->K) return fail(SVDQ_ERR_INVALID_ARG, "the up layer's N must be the down layer's K");
  if (down->K % 256) return fail(SVDQ_ERR_UNSUPPORTED, "the fused MLP block needs the down layer's K % 256 == 0");
  if (down->RP != kMlpDownRP)
    return fail(SVDQ_ERR_UNSUPPORTED, "the fused MLP block needs a down-layer branch of 1..32 columns");
  if (up->device != down->device) return fail(SVDQ_ERR_INVALID_ARG, "the layers live on different devices");
  return SVDQ_OK;
}

svdq_status mlp_impl(svdq_layer* up, svdq_layer* down, const void* X, int M, void* Y, void* workspace,
                     size_t ws_bytes, void* stream, void* const* events) {
  if (svdq_status e = check_mlp(up, down)) return e;
  if (!X || !Y || !workspace || M < 1) return fail(SVDQ_ERR_INVALID_ARG, "NULL pointer or M < 1");
  if (!aligned16(X) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(SVDQ_ERR_INVALID_ARG, "X/Y must be 16-byte and the workspace 256-byte aligned");
  if (svdq_status e = check_layer_device(up)) return e;
  const MlpLayout l = mlp_layout(up, down, M);
  if (static_cast<long long>(l.tiles + 1) * l.pairs >= (1LL << 31))
    return fail(SVDQ_ERR_INVALID_ARG, "M exceeds the rows the fused MLP block supports");
  if (ws_bytes < l.total) return fail(SVDQ_ERR_INVALID_ARG, "workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint8_t* dbase = base + l.down_off;
  uint8_t* codes_d = dbase + l.down.codes;
  uint8_t* scales_d = dbase + l.down.scales;
  __nv_bfloat16* T_d = reinterpret_cast<__nv_bfloat16*>(dbase + l.down.T);
  float* tpart = reinterpret_cast<float*>(base + l.tpart_off);
  __nv_bfloat16* T_lo = up->RP > 0 ? reinterpret_cast<__nv_bfloat16*>(base + l.tlo_off) : nullptr;
  // the down layer's factor as the fused epilogue loads it: each CTA of a pair its 16 rows
  if (!down->mlp_maps_ready) {
    if (!make_map(&down->map_l1h_half, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, down->L1sTh, down->K, down->RP,
                  static_cast<uint64_t>(down->K) * 2, 64, kMlpDownRP / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&down->map_l1l_half, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, down->L1sTl, down->K, down->RP,
                  static_cast<uint64_t>(down->K) * 2, 64, kMlpDownRP / 2, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (down-layer factor) failed");
    down->mlp_maps_ready = true;
  }
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[0]), st));
  svdq_status e = launch_k1(up, X, M, base + l.up.codes, base + l.up.scales,
                            reinterpret_cast<__nv_bfloat16*>(base + l.up.T), reinterpret_cast<float*>(base + l.up.Tpart),
                            l.up, nullptr, st, T_lo);
  if (e) return e;
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[1]), st));
  MlpDownParams mp{};
  mp.K = down->K;
  mp.M_pad = l.down.M_pad;
  mp.inv_s = down->inv_s;
  mp.codes = codes_d;
  mp.scales = scales_d;
  mp.g_x = down->g_x;
  mp.denom = down->denom;
  mp.tpart = tpart;
  mp.slots = l.slots;
  GemmMaps extra{};
  extra.l1h_down = down->map_l1h_half;
  extra.l1l_down = down->map_l1l_half;
  if ((e = gemm_stage(up, M, nullptr, base + l.up.codes, base + l.up.scales,
                      reinterpret_cast<__nv_bfloat16*>(base + l.up.T), T_lo, &mp, &extra, st)))
    return e;
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[2]), st));
  cudaError_t ce = launch_mlp_t_reduce(tpart, l.down.M_pad, l.slots, l.tiles, l.n_blocks, l.pairs, down->t_scale, T_d, st);
  if (ce != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("T reduction: ") + cudaGetErrorString(ce));
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[3]), st));
  if ((e = gemm_stage(down, M, Y, codes_d, scales_d, T_d, nullptr, nullptr, nullptr, st))) return e;
  if (events) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(events[4]), st));
  return SVDQ_OK;
}

}  // namespace

extern "C" {

svdq_status svdq_linear_forward(svdq_layer_t h, const void* X, int M, void* Y, void* workspace, size_t ws_bytes,
                                void* stream) {
  return forward_impl(h, X, M, Y, workspace, ws_bytes, nullptr, stream, nullptr);
}

svdq_status svdq_mlp_workspace_size(svdq_layer_t up, svdq_layer_t down, int M, size_t* bytes) {
  if (svdq_status e = check_mlp(up, down)) return e;
  if (!bytes || M < 1) return fail(SVDQ_ERR_INVALID_ARG, "bad workspace query");
  *bytes = mlp_layout(up, down, M).total;
  return SVDQ_OK;
}

svdq_status svdq_mlp_workspace_layout(svdq_layer_t up, svdq_layer_t down, int M, size_t* offsets) {
  if (svdq_status e = check_mlp(up, down)) return e;
  if (!offsets || M < 1) return fail(SVDQ_ERR_INVALID_ARG, "bad layout query");
  const MlpLayout l = mlp_layout(up, down, M);
  offsets[0] = l.down_off + l.down.codes;
  offsets[1] = l.down_off + l.down.scales;
  offsets[2] = l.down_off + l.down.T;
  return SVDQ_OK;
}

svdq_status svdq_mlp_forward(svdq_layer_t up, svdq_layer_t down, const void* X, int M, void* Y, void* workspace,
                             size_t ws_bytes, void* stream) {
  return mlp_impl(up, down, X, M, Y, workspace, ws_bytes, stream, nullptr);
}

svdq_status svdq_mlp_forward_profiled(svdq_layer_t up, svdq_layer_t down, const void* X, int M, void* Y,
                                      void* workspace, size_t ws_bytes, void* stream, void* const* events) {
  if (!events) return fail(SVDQ_ERR_INVALID_ARG, "five events needed");
  for (int i = 0; i < 5; ++i)
    if (!events[i]) return fail(SVDQ_ERR_INVALID_ARG, "five events needed");
  return mlp_impl(up, down, X, M, Y, workspace, ws_bytes, stream, events);
}

svdq_status svdq_linear_forward_masked(svdq_layer_t h, const void* X, int M, void* Y, void* workspace,
                                       size_t ws_bytes, const uint32_t* row_adapter_mask, void* stream) {
  if (!row_adapter_mask) return fail(SVDQ_ERR_INVALID_ARG, "row_adapter_mask is NULL (use svdq_linear_forward)");
  return forward_impl(h, X, M, Y, workspace, ws_bytes, row_adapter_mask, stream, nullptr);
}

svdq_status svdq_linear_forward_profiled(svdq_layer_t h, const void* X, int M, void* Y, void* workspace,
                                         size_t ws_bytes, void* stream, void* const* events) {
  if (!events || !events[0] || !events[1] || !events[2]) return fail(SVDQ_ERR_INVALID_ARG, "three events needed");
  return forward_impl(h, X, M, Y, workspace, ws_bytes, nullptr, stream, events);
}

svdq_status svdq_quantize_activations(svdq_layer_t h, const void* X, int M, void* codes, void* scales, void* T,
                                      void* stream) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (!X || !codes || !scales || (!T && h->RP > 0) || M < 1) return fail(SVDQ_ERR_INVALID_ARG, "NULL pointer or M < 1");
  if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || (T && !aligned16(T)))
    return fail(SVDQ_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (svdq_status e = check_layer_device(h)) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(h, M);
  // float partials over the K shares: a scratch buffer of this call's own
  float* Tpart = nullptr;
  if (w.split > 1 && h->RP > 0) {
    if (injected_alloc_failure()) return fail(SVDQ_ERR_OOM, "device allocation failed (injected by the test hook)");
    cudaError_t ce = cudaMallocAsync(reinterpret_cast<void**>(&Tpart), w.total - w.Tpart, st);
    if (ce != cudaSuccess) return fail(SVDQ_ERR_OOM, std::string("T partials: ") + cudaGetErrorString(ce));
  }
  svdq_status e =
      launch_k1(h, X, M, static_cast<uint8_t*>(codes), scales, static_cast<__nv_bfloat16*>(T), Tpart, w, nullptr, st);
  if (Tpart) cudaFreeAsync(Tpart, st);
  return e;
}

svdq_status svdq_attach_lora(svdq_layer_t h, const void* A, const void* B, int r_l, float scale, void* stream,
                             int* slot_out) {
  if (slot_out) *slot_out = -1;
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (!A || !B || r_l < 1) return fail(SVDQ_ERR_INVALID_ARG, "bad LoRA arguments");
  if (h->rank + r_l > 256) return fail(SVDQ_ERR_INVALID_ARG, "rank + r_l exceeds 256");
  if (!std::isfinite(scale)) return fail(SVDQ_ERR_INVALID_ARG, "scale must be finite");
  if (!aligned16(A) || !aligned16(B)) return fail(SVDQ_ERR_INVALID_ARG, "A and B must be 16-byte aligned");
  int slot = -1;
  for (int a = 0; a < kMaxAdapters && slot < 0; ++a)
    if (h->adapters[a].rank == 0) slot = a;
  if (slot < 0) return fail(SVDQ_ERR_INVALID_ARG, "every adapter slot is taken (detach one first)");
  if (svdq_status e = check_layer_device(h)) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  svdq_layer::Adapter ad;
  ad.rank = r_l;
  svdq_status e;
  if ((e = dalloc(&ad.F, static_cast<size_t>(h->K) * r_l * 2))) return e;
  if ((e = dalloc(&ad.G, static_cast<size_t>(r_l) * h->N * 2))) return cudaFree(ad.F), e;
  if (launch_lora_factors(static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), h->K, h->N, r_l,
                          scale, h->s, ad.F, ad.G, st) != cudaSuccess) {
    cudaFree(ad.F);
    cudaFree(ad.G);
    return fail(SVDQ_ERR_CUDA, "LoRA factor launch failed");
  }
  h->adapters[slot] = ad;
  if ((e = assemble_branch(h, st))) {
    cudaStreamSynchronize(st);
    cudaFree(ad.F);
    cudaFree(ad.G);
    h->adapters[slot] = svdq_layer::Adapter{};
    return e;
  }
  if (slot_out) *slot_out = slot;
  return SVDQ_OK;
}

svdq_status svdq_detach_lora(svdq_layer_t h, int slot, void* stream) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (slot < 0 || slot >= kMaxAdapters || h->adapters[slot].rank == 0)
    return fail(SVDQ_ERR_INVALID_ARG, "no adapter in slot " + std::to_string(slot));
  if (svdq_status e = check_layer_device(h)) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const svdq_layer::Adapter ad = h->adapters[slot];
  h->adapters[slot] = svdq_layer::Adapter{};
  if (svdq_status e = assemble_branch(h, st)) {
    h->adapters[slot] = ad;  // nothing was swapped: the layer keeps the adapter
    return e;
  }
  cudaFree(ad.F);
  cudaFree(ad.G);
  return SVDQ_OK;
}

svdq_status svdq_layer_get_info(svdq_layer_t h, svdq_layer_info* info) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (!info) return fail(SVDQ_ERR_INVALID_ARG, "info is NULL");
  info->K = h->K;
  info->N = h->N;
  info->rank = h->rank;
  info->rank_pad = h->RP;
  info->base_rank = h->base_rank;
  info->flags = h->cfg.flags;
  info->adapter_slots = 0;
  for (int a = 0; a < kMaxAdapters; ++a) {
    if (h->adapters[a].rank) info->adapter_slots |= 1u << a;
    info->adapter_col_start[a] = h->col_start[a];
  }
  info->adapter_col_start[kMaxAdapters] = h->col_start[kMaxAdapters];
  info->fmt = h->fmt;
  info->alpha = h->cfg.alpha;
  info->g_x = h->g_x;
  info->g_w = h->g_w;
  info->t_scale = h->t_scale;
  return SVDQ_OK;
}

svdq_status svdq_export_weights(svdq_layer_t h, void* blob, size_t* bytes, void* stream) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "bytes is NULL");
  const int K = h->K, N = h->N, r = h->rank;
  const bool i4 = h->fmt == SVDQ_INT4_G64;
  svdq_blob_header hd{};
  hd.magic = 0x51445653u;
  hd.version = 1;
  hd.fmt = h->fmt;
  hd.K = K;
  hd.N = N;
  hd.rank = r;
  hd.alpha = h->cfg.alpha;
  hd.g_x = h->g_x;
  hd.g_w = h->g_w;
  size_t off = align256(sizeof(svdq_blob_header));
  auto take = [&](size_t n) {
    size_t o = off;
    off = align256(off + n);
    return static_cast<uint64_t>(o);
  };
  hd.off_s = take(K * 4);
  hd.off_inv_s = take(K * 4);
  hd.off_L1 = take(static_cast<size_t>(K) * r * 2);
  hd.off_L2 = take(static_cast<size_t>(r) * N * 2);
  hd.off_codes = take(static_cast<size_t>(N) * K / 2);
  hd.off_scales = take(i4 ? static_cast<size_t>(N) * (K / 64) * 4 : static_cast<size_t>(N) * (K / 16));
  hd.off_bias = take(N * 2);
  hd.total = off;
  if (!blob) {
    *bytes = off;
    return SVDQ_OK;
  }
  if (*bytes < off) return fail(SVDQ_ERR_INVALID_ARG, "blob too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(blob);
  std::memset(b, 0, off);
  std::memcpy(b, &hd, sizeof(hd));
  std::vector<uint16_t> l1t(static_cast<size_t>(h->RP) * K), l2t(static_cast<size_t>(h->N_pad) * h->RP);
  const size_t cbytes = i4 ? static_cast<size_t>(h->N_pad) * K : static_cast<size_t>(h->N_pad) * K / 2;
  const size_t sbytes = i4 ? static_cast<size_t>(K / 64) * h->N_pad * 4 : static_cast<size_t>(h->N_pad / 128) * (K / 64) * 512;
  std::vector<uint8_t> codes(cbytes), scales(sbytes);
  CUDA_TRY(cudaMemcpyAsync(b + hd.off_s, h->s, K * 4, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaMemcpyAsync(b + hd.off_inv_s, h->inv_s, K * 4, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaMemcpyAsync(b + hd.off_bias, h->bias, N * 2, cudaMemcpyDeviceToHost, st));
  if (h->RP > 0) {
    CUDA_TRY(cudaMemcpyAsync(l1t.data(), h->L1T, l1t.size() * 2, cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaMemcpyAsync(l2t.data(), h->L2T, l2t.size() * 2, cudaMemcpyDeviceToHost, st));
  }
  CUDA_TRY(cudaMemcpyAsync(codes.data(), h->wcodes, cbytes, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaMemcpyAsync(scales.data(), h->wscales, sbytes, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  uint16_t* L1 = reinterpret_cast<uint16_t*>(b + hd.off_L1);
  uint16_t* L2 = reinterpret_cast<uint16_t*>(b + hd.off_L2);
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < r; ++j) L1[static_cast<size_t>(k) * r + j] = l1t[static_cast<size_t>(j) * K + k];
  for (int j = 0; j < r; ++j)
    for (int n = 0; n < N; ++n) L2[static_cast<size_t>(j) * N + n] = l2t[static_cast<size_t>(n) * h->RP + j];
  uint8_t* C = b + hd.off_codes;
  if (i4) {
    // E4M3 bytes of the integers -8..7 back to two's-complement nibbles
    auto to_int = [](uint8_t e) -> int {
      const int mag_code = e & 0x7F;
      int mag = 0;
      switch (mag_code) {
        case 0x00: mag = 0; break;
        case 0x38: mag = 1; break;
        case 0x40: mag = 2; break;
        case 0x44: mag = 3; break;
        case 0x48: mag = 4; break;
        case 0x4A: mag = 5; break;
        case 0x4C: mag = 6; break;
        case 0x4E: mag = 7; break;
        case 0x50: mag = 8; break;
        default: mag = 0; break;
      }
      return (e & 0x80) ? -mag : mag;
    };
    for (int n = 0; n < N; ++n)
      for (int k = 0; k < K; k += 2) {
        const int q0 = to_int(codes[static_cast<size_t>(n) * K + k]);
        const int q1 = to_int(codes[static_cast<size_t>(n) * K + k + 1]);
        C[static_cast<size_t>(n) * (K / 2) + k / 2] = static_cast<uint8_t>((q0 & 0xF) | ((q1 & 0xF) << 4));
      }
    float* S = reinterpret_cast<float*>(b + hd.off_scales);
    const float* sw = reinterpret_cast<const float*>(scales.data());
    for (int n = 0; n < N; ++n)
      for (int g = 0; g < K / 64; ++g) S[static_cast<size_t>(n) * (K / 64) + g] = sw[static_cast<size_t>(g) * h->N_pad + n];
  } else {
    std::memcpy(C, codes.data(), static_cast<size_t>(N) * K / 2);
    uint8_t* S = b + hd.off_scales;
    for (int n = 0; n < N; ++n)
      for (int i = 0; i < K / 16; ++i) {
        const size_t atom = static_cast<size_t>(n / 128) * (K / 64) + i / 4;
        S[static_cast<size_t>(n) * (K / 16) + i] = scales[atom * 512 + (n % 32) * 16 + ((n / 32) % 4) * 4 + i % 4];
      }
  }
  *bytes = off;
  return SVDQ_OK;
}

svdq_status svdq_device_status(svdq_layer_t h, void* stream) {
  if (check_layer(h)) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  CUDA_TRY(cudaMemcpyAsync(&v, h->status, 4, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  CUDA_TRY(cudaMemsetAsync(h->status, 0, 4, st));
  if (v == kDevTimeout) return fail(SVDQ_ERR_DEVICE_TIMEOUT, "a kernel gave up a pipeline wait");
  return SVDQ_OK;
}

svdq_status svdq_destroy(svdq_layer_t h) {
  if (!h) return SVDQ_OK;
  cudaDeviceSynchronize();
  free_layer(h);
  return SVDQ_OK;
}

void svdq_debug_fail_allocation(long long index) { g_fail_alloc_at.store(index < 0 ? -1 : index); }

svdq_status svdq_selftest_bounded_wait(unsigned long long limit_ns, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  svdq_status e;
  if ((e = dalloc(&status, 16))) return e;
  int v = -1;
  cudaError_t ce = cudaMemsetAsync(status, 0xFF, 4, st);
  if (ce == cudaSuccess) ce = launch_wait_selftest(status, limit_ns, st);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(&v, status, 4, cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  cudaFree(status);
  if (ce != cudaSuccess) return fail(SVDQ_ERR_CUDA, cudaGetErrorString(ce));
  if (v == kDevTimeout) return fail(SVDQ_ERR_DEVICE_TIMEOUT, "bounded wait gave up as designed");
  return SVDQ_OK;
}

}  // extern "C"
