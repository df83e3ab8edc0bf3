// The 4-bit weight-only baseline (W4A16) that the SVDQuant abstract compares
// against ("3.0x speedup over the 4-bit weight-only quantized baseline").
//
// The weights are quantized on their own, with no smoothing and no low-rank
// branch, by the same symmetric INT4 group-64 quantizer the W4A4 layer uses
// (scale = amax / 7 per output column and 64-element group along K); the
// activations stay bf16:
//   w_deq[n, k] = bf16( fp32(q[n, k] * scale[n, k / 64]) )
//   Y = X w_deq^T + b            (fp32 accumulation, one bf16 store)
// The weights stay packed in HBM (two codes per byte) and are dequantized into
// shared memory tile by tile, so every forward reads 4-bit weights, as a
// weight-only kernel does.
//
// Kernel: one CTA per 128 x 256 output tile, 64-wide K chunks (one group).
//   warp 0      producer: per chunk, the X tile [128 x 64] bf16 (TMA, 128-byte
//               swizzle), the packed codes of the tile's 256 columns [256 x 32 B]
//               (TMA) and their 256 group scales (bulk copy), 4-stage ring;
//   warps 2-17  dequantizers: thread t owns column t % 256 and half t / 256 of
//               the chunk (32 codes): integer code -> float (exact, by the
//               2^23 bit trick), times the scale, rounded to bf16, written in
//               the tcgen05 K-major 128-byte-swizzled layout into one of two
//               B-operand buffers; after the last chunk the same warps run the
//               epilogue (TMEM -> registers, + bias, bf16 store);
//   warp 1      MMA issuer: tcgen05 kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//               M 128, N 256, four K-16 steps per chunk.
#include <cstdint>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace svdq {
void set_last_error(const std::string& msg);
}

using namespace svdq;

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;  // one quantization group per chunk
constexpr int kStages = 4;
constexpr int kBBufs = 2;
constexpr int kDqWarps = 16;
constexpr int kThreads = (2 + kDqWarps) * 32;

struct SmemW {
  static constexpr int kX = kBM * kBK * 2;  // 16 KB
  static constexpr int kC = kBN * kBK / 2;  // 8 KB of packed codes
  static constexpr int kS = kBN * 4;        // 1 KB of scales
  static constexpr int kStage = kX + kC + kS;
  static constexpr int kBOff = kStages * kStage;
  static constexpr int kB = kBN * kBK * 2;  // 32 KB bf16 operand
  static constexpr int kBarOff = kBOff + kBBufs * kB;
  static constexpr int kTotal = kBarOff + 256 + 1024;
};
static_assert(SmemW::kTotal <= 232448, "shared memory budget");
static_assert(SmemW::kStage % 1024 == 0 && SmemW::kBOff % 1024 == 0, "swizzled tiles start 1 KB-aligned");

struct W4Params {
  int M, N, K, N_pad;
  __nv_bfloat16* Y;
  const __nv_bfloat16* bias;  // [N_pad]
  const float* scales;        // [K/64][N_pad]
  int* status;
};
struct W4Maps {
  CUtensorMap x;      // X [M, K] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap codes;  // codes [N_pad, K/2] u8, box {32, 256}
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two's-complement nibble -> exact float: flipping bit 3 gives q + 8 in
// 0..15; placed in the mantissa of 2^23 that is 2^23 + q + 8, and subtracting
// 2^23 + 8 leaves q exactly.
__device__ __forceinline__ float nibble_to_float(uint32_t word, int i) {
  const uint32_t u = ((word >> (4 * i)) & 0xFu) ^ 0x8u;
  return __fsub_rn(__uint_as_float(0x4B000000u | u), 8388616.0f);
}

__global__ void __launch_bounds__(kThreads, 1) gemm_w4a16_kernel(const W4Params p, const __grid_constant__ W4Maps maps) {
  using L = SmemW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* bready = empty + kStages;
  uint64_t* bfree = bready + kBBufs;
  uint64_t* acc_full = bfree + kBBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = p.N_pad / kBN;
  const int mb = blockIdx.x / n_blocks, nb = blockIdx.x % n_blocks;
  const int m0 = mb * kBM, n0 = nb * kBN;
  const int nk = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDqWarps + 1);
    }
    for (int b = 0; b < kBBufs; ++b) {
      mbar_init(&bready[b], kDqWarps);
      mbar_init(&bfree[b], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&maps.x);
      prefetch_tensormap(&maps.codes);
      int j = 0;
      for (; j < nk; ++j) {
        const int s = j % kStages;
        if (!mbar_wait(&empty[s], ((j / kStages) & 1) ^ 1, abort_flag, p.status)) break;
        uint8_t* st = smem + s * L::kStage;
        mbar_arrive_expect_tx(&full[s], L::kX + L::kC + L::kS);
        tma_load_2d(st, &maps.x, &full[s], j * kBK, m0);
        tma_load_2d(st + L::kX, &maps.codes, &full[s], j * (kBK / 2), n0);
        bulk_load(st + L::kX + L::kC, p.scales + static_cast<size_t>(j) * p.N_pad + n0, L::kS, &full[s]);
      }
      if (j < nk) {  // gave up: let the copies in flight land before exiting
        volatile int no_abort = 0;
        for (int i = max(0, j - kStages); i < j; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, &no_abort, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kBM, kBN);
      for (int j = 0; j < nk; ++j) {
        const int s = j % kStages, b = j % kBBufs;
        if (!mbar_wait(&full[s], (j / kStages) & 1, abort_flag, p.status)) break;
        if (!mbar_wait(&bready[b], (j / kBBufs) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + s * L::kStage);
        const uint32_t bw = smem_u32(smem + L::kBOff + b * L::kB);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16(tmem, smem_desc(xa + 32 * ks, 16, 1024, kSw128), smem_desc(bw + 32 * ks, 16, 1024, kSw128), idesc,
                  (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
        tc_commit(&bfree[b]);
      }
      tc_commit(acc_full);  // every MMA issued above has completed when this arrives
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ dequantize W into the B operand
    const int t = threadIdx.x - 64;  // 0..511
    const int n = t & (kBN - 1);      // column of the tile = row of the K-major B operand
    const int h = t >> 8;             // which half of the chunk's 64 K
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      const int s = j % kStages, b = j % kBBufs;
      ok = mbar_wait(&full[s], (j / kStages) & 1, abort_flag, p.status);
      if (!ok) break;
      const uint8_t* st = smem + s * L::kStage;
      const uint4 c = *reinterpret_cast<const uint4*>(st + L::kX + n * 32 + h * 16);
      const float sc = reinterpret_cast<const float*>(st + L::kX + L::kC)[n];
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // codes and scale are in registers
      if (j >= kBBufs) {
        ok = mbar_wait(&bfree[b], ((j / kBBufs) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
      }
      const uint32_t w[4] = {c.x, c.y, c.z, c.w};
      uint8_t* bt = smem + L::kBOff + b * L::kB;
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // 8 codes (16 bytes of bf16) per swizzle chunk
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = __fmul2_rn(make_float2(nibble_to_float(w[q], 2 * e), nibble_to_float(w[q], 2 * e + 1)),
                                      make_float2(sc, sc));
          o[e] = pack_bf16x2(v.x, v.y);
        }
        const int chunk = 4 * h + q;  // 16-byte chunk of the 128-byte row
        *reinterpret_cast<uint4*>(bt + n * 128 + ((chunk ^ (n & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&bready[b]);
    }
    // ------------------------------------------------ epilogue
    if (ok) {
      volatile int no_abort = 0;
      ok = mbar_wait(acc_full, 0, &no_abort, nullptr) && !*abort_flag;
    }
    tc_fence_after();
    const int ew = warp - 2;         // 0..15
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int col0 = (ew >> 2) * 64;
    const int row = m0 + 32 * q + lane;
    if (ok) {
#pragma unroll 1
      for (int cc = 0; cc < 64; cc += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + col0 + cc, r);
        tmem_ld_wait();
        const int nbase = n0 + col0 + cc;
        if (row < p.M) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int nn = nbase + 8 * v;
            if (nn < p.N) {
              const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + nn));
              const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                o[e] = pack_bf16x2(__uint_as_float(r[8 * v + 2 * e]) + __uint_as_float(bb[e] << 16),
                                   __uint_as_float(r[8 * v + 2 * e + 1]) + __uint_as_float(bb[e] & 0xFFFF0000u));
              *reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(row) * p.N + nn) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Symmetric INT4 group-64 quantization of W [K, N] bf16 per output column:
// thread per (n, group). Codes as two's-complement nibbles [N_pad, K/2]
// (element 2j in bits 3:0), scales float [K/64][N_pad]; scale = amax/7,
// q = rint(fp32(w * (7 / amax))), both IEEE round-to-nearest; an all-zero
// group has scale 0 and codes 0.
__global__ void quant_w4a16_kernel(const __nv_bfloat16* W, int K, int N, int N_pad, uint8_t* codes, float* scales) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (n >= N) return;
  float v[64];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    v[i] = __bfloat162float(W[static_cast<size_t>(g * 64 + i) * N + n]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float scale = 0.f;
  if (amax > 0.f) {
    scale = __fdiv_rn(amax, 7.0f);
    const float inv = __fdiv_rn(7.0f, amax);
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const int q = min(7, max(-8, __float2int_rn(__fmul_rn(v[i], inv))));
      w[i >> 3] |= (static_cast<uint32_t>(q) & 0xFu) << (4 * (i & 7));
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(n) * (K / 2) + g * 32);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  scales[static_cast<size_t>(g) * N_pad + n] = scale;
}

}  // namespace

struct svdq_w4a16 {
  int device = 0;
  int K = 0, N = 0, N_pad = 0;
  uint8_t* codes = nullptr;      // [N_pad, K/2]
  float* scales = nullptr;       // [K/64][N_pad]
  __nv_bfloat16* bias = nullptr; // [N_pad]
  int* status = nullptr;
  CUtensorMap map_codes{};
  const void* x_key = nullptr;   // last X the X map was built for
  int x_rows = -1;
  CUtensorMap map_x{};
};

namespace {

svdq_status w4_fail(svdq_status st, const std::string& msg) {
  set_last_error(msg);
  return st;
}

void w4_free(svdq_w4a16* h) {
  if (!h) return;
  cudaFree(h->codes);
  cudaFree(h->scales);
  cudaFree(h->bias);
  cudaFree(h->status);
  delete h;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" {

svdq_status svdq_w4a16_prepare(const void* W, const void* bias, int K, int N, void* stream, svdq_w4a16_t* out) {
  if (!out) return w4_fail(SVDQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!W || K <= 0 || K % 128 || N <= 0 || N % 16) return w4_fail(SVDQ_ERR_INVALID_ARG, "bad W4A16 shape or NULL W");
  if (!al16(W) || (bias && !al16(bias))) return w4_fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  svdq_w4a16* h = new svdq_w4a16();
  cudaGetDevice(&h->device);
  h->K = K;
  h->N = N;
  h->N_pad = (N + 255) / 256 * 256;
  const size_t cb = static_cast<size_t>(h->N_pad) * K / 2, sb = static_cast<size_t>(K / 64) * h->N_pad * 4;
  if (cudaMalloc(&h->codes, cb) != cudaSuccess || cudaMalloc(&h->scales, sb) != cudaSuccess ||
      cudaMalloc(&h->bias, h->N_pad * 2) != cudaSuccess || cudaMalloc(&h->status, 16) != cudaSuccess) {
    cudaGetLastError();
    w4_free(h);
    return w4_fail(SVDQ_ERR_OOM, "W4A16 buffers: cudaMalloc failed");
  }
  cudaError_t e = cudaMemsetAsync(h->codes, 0, cb, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->scales, 0, sb, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->bias, 0, h->N_pad * 2, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->status, 0, 16, st);
  if (e == cudaSuccess && bias) e = cudaMemcpyAsync(h->bias, bias, N * 2, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) {
    quant_w4a16_kernel<<<dim3((N + 127) / 128, K / 64), 128, 0, st>>>(static_cast<const __nv_bfloat16*>(W), K, N,
                                                                       h->N_pad, h->codes, h->scales);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    w4_free(h);
    return w4_fail(SVDQ_ERR_CUDA, std::string("W4A16 prepare: ") + cudaGetErrorString(e));
  }
  if (!make_map(&h->map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, h->codes, K / 2, h->N_pad, K / 2, 32, 256,
                CU_TENSOR_MAP_SWIZZLE_NONE)) {
    w4_free(h);
    return w4_fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (W4A16 codes) failed");
  }
  *out = h;
  return SVDQ_OK;
}

svdq_status svdq_w4a16_forward(svdq_w4a16_t h, const void* X, int M, void* Y, void* stream) {
  if (!h) return w4_fail(SVDQ_ERR_INVALID_ARG, "W4A16 layer is NULL");
  if (!X || !Y || M < 1) return w4_fail(SVDQ_ERR_INVALID_ARG, "NULL pointer or M < 1");
  if (!al16(X) || !al16(Y)) return w4_fail(SVDQ_ERR_INVALID_ARG, "X/Y must be 16-byte aligned");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device)
    return w4_fail(SVDQ_ERR_INVALID_ARG, "the current device is not the layer's device");
  if (h->x_key != X || h->x_rows != M) {
    h->x_key = nullptr;
    if (!make_map(&h->map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, h->K, M, static_cast<uint64_t>(h->K) * 2, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return w4_fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (W4A16 X) failed");
    h->x_key = X;
    h->x_rows = M;
  }
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(gemm_w4a16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemW::kTotal);
  });
  if (e != cudaSuccess) return w4_fail(SVDQ_ERR_CUDA, cudaGetErrorString(e));
  W4Params p{M, h->N, h->K, h->N_pad, static_cast<__nv_bfloat16*>(Y), h->bias, h->scales, h->status};
  W4Maps maps{h->map_x, h->map_codes};
  const int tiles = ((M + kBM - 1) / kBM) * (h->N_pad / kBN);
  gemm_w4a16_kernel<<<tiles, kThreads, SmemW::kTotal, static_cast<cudaStream_t>(stream)>>>(p, maps);
  e = cudaGetLastError();
  if (e != cudaSuccess) return w4_fail(SVDQ_ERR_CUDA, std::string("W4A16 kernel: ") + cudaGetErrorString(e));
  return SVDQ_OK;
}

svdq_status svdq_w4a16_export(svdq_w4a16_t h, void* codes, void* scales, void* stream) {
  if (!h || !codes || !scales) return w4_fail(SVDQ_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpy2DAsync(codes, h->K / 2, h->codes, h->K / 2, h->K / 2, h->N, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(scales, h->N * 4, h->scales, h->N_pad * 4, h->N * 4, h->K / 64, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return w4_fail(SVDQ_ERR_CUDA, cudaGetErrorString(e));
  return SVDQ_OK;
}

svdq_status svdq_w4a16_destroy(svdq_w4a16_t h) {
  if (!h) return SVDQ_OK;
  cudaDeviceSynchronize();
  w4_free(h);
  return SVDQ_OK;
}

}  // extern "C"
