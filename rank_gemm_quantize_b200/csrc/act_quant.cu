// K1: activation smoothing + 4-bit group quantization + low-rank down-projection.
//
// SVDQuant ("SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit
// Diffusion Models", abstract; msModelSlim SVDQuant entry, section 2.3, the
// dual-path output equation) runs, per layer and per input row x:
//   x_hat = x diag(s)^-1                      (the migration identity, eq. 1)
//   Q(x_hat): 4-bit codes + one scale per group along K
//   T     = x_hat L1                          (the branch input X diag(s)^-1 V)
// This kernel reads every X element from HBM once and produces all three in
// the same pass.
//
// Work split: a thread-block cluster of S CTAs owns 128 rows; CTA r of the
// cluster walks its 1/S share of K in 64-column chunks (S is chosen so the
// grid covers the SMs once). Per chunk:
//   * warp 16 (one thread) streams the X tile [128 x 64] and the L1^T slice
//     [RP x 64] into a shared-memory ring with TMA (128-byte swizzle);
//   * warps 0-15 (8 rows each) smooth, quantize, store codes and scales, and
//     write x_hat as a bf16 high part and a bf16 remainder straight into a
//     tcgen05 K-major operand buffer;
//   * the same thread of warp 16 then issues tcgen05 kind::f16 MMAs
//     (M = 128, N = RP, bf16 x bf16 -> fp32) of hi and lo against L1 into a
//     TMEM accumulator, so T carries float32-level accuracy before its store.
// At the end the S partial T tiles are reduced through distributed shared
// memory in a fixed rank order (deterministic), scaled and stored as bf16.
//
// Numerics of the quantizer match the CPU oracle operation by operation:
// every product and quotient is a single IEEE round-to-nearest operation
// (__fmul_rn / __fdiv_rn, no FMA contraction), rint is round-half-even, and the
// E4M3 / E2M1 encodings use the hardware cvt.rn.satfinite conversions.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kRows = 128;     // rows per cluster (one tcgen05 M)
constexpr int kQWarps = 16;    // quantizing warps, 8 rows each
constexpr int kThreads = (kQWarps + 1) * 32;
constexpr int kChunk = 64;     // columns per chunk (one 128-byte swizzle atom of bf16)
constexpr int kRedCols = 64;   // columns per cluster-reduction pass

template <int RP>
struct K1Shape {
  static constexpr int kStages = RP <= 64 ? 4 : (RP <= 128 ? 3 : 2);
  static constexpr int kX = kRows * 128;             // X tile of a chunk (bf16, 64 cols)
  static constexpr int kL = RP * 128;                // L1^T slice of a chunk
  static constexpr int kS = 1024;                    // inv_s slice of a chunk (256 B used, 1 KB keeps alignment)
  static constexpr int kStage = kX + kL + kS;
  static constexpr int kA = 2 * kRows * 128;         // hi + lo MMA operand of a chunk
  static constexpr int kAOff = kStages * kStage;
  static constexpr int kRedOff = kAOff + 2 * kA;
  static constexpr int kRedW = RP < kRedCols ? RP : kRedCols;
  static constexpr int kRed = kRows * kRedW * 4;
  static constexpr int kBarOff = kRedOff + kRed;
  static constexpr int kTotal = kBarOff + 256 + 1024;
  static constexpr uint32_t kTmemCols = RP <= 32 ? 32 : (RP <= 64 ? 64 : (RP <= 128 ? 128 : 256));
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_peer_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Quantize 8 consecutive smoothed values of one row (this lane's share of a
// group), store the codes, and the group scale from one lane per group.
template <int FMT>
__device__ __forceinline__ void quantize8(const float (&v)[8], const ActQuantParams& p, int row, int k, int cs) {
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
  if (FMT == SVDQ_INT4_G64) {
    // group of 64 = the 8 lanes sharing (lane >> 3)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    float scale = 0.f;
    uint32_t lo = 0, hi = 0;
    if (amax > 0.f) {
      scale = __fdiv_rn(amax, 7.0f);
      const float inv = __fdiv_rn(7.0f, amax);
      // |v| <= amax and inv <= (7 / amax)(1 + 2^-24), so |v * inv| rounds to at
      // most 7: rint already lands in [-7, 7] and the [-8, 7] clamp never acts.
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 pr = __fmul2_rn(make_float2(v[j], v[j + 1]), make_float2(inv, inv));
        q[j] = rintf(pr.x);
        q[j + 1] = rintf(pr.y);
      }
      lo = cvt_e4m3x2(q[0], q[1]) | (cvt_e4m3x2(q[2], q[3]) << 16);
      hi = cvt_e4m3x2(q[4], q[5]) | (cvt_e4m3x2(q[6], q[7]) << 16);
    }
    uint8_t* dst = p.codes + static_cast<size_t>(row) * p.K + k;
    *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
    if (cs == 0) reinterpret_cast<float*>(p.scales)[static_cast<size_t>(k >> 6) * p.M_pad + row] = scale;
  } else {
    // group of 16 = this lane and its neighbour (lane ^ 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const float r = __fdiv_rn(amax, p.denom);
    const uint32_t sb = cvt_e4m3x2(r, 0.f) & 0xFFu;
    const float eff = __fmul_rn(e4m3_to_float(sb), p.g_x);
    uint32_t codes = 0;
    if (eff != 0.f) {
      const float inv = __frcp_rn(eff);
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 pr = __fmul2_rn(make_float2(v[j], v[j + 1]), make_float2(inv, inv));
        q[j] = pr.x;
        q[j + 1] = pr.y;
      }
      codes = cvt_e2m1x8(q);
    }
    uint8_t* dst = p.codes + static_cast<size_t>(row) * (p.K >> 1) + (k >> 1);
    *reinterpret_cast<uint32_t*>(dst) = codes;
    if ((cs & 1) == 0) {
      const int sf = k >> 4;  // scale index along the row
      const size_t atom = static_cast<size_t>(row >> 7) * (p.K >> 6) + (sf >> 2);
      const int off = (row & 31) * 16 + ((row >> 5) & 3) * 4 + (sf & 3);
      reinterpret_cast<uint8_t*>(p.scales)[atom * 512 + off] = static_cast<uint8_t>(sb);
    }
  }
}

template <int FMT, int RP>
__global__ void __launch_bounds__(kThreads, 1)
    act_quant_kernel(const ActQuantParams p, const __grid_constant__ ActQuantMaps maps) {
  using S = K1Shape<RP>;
  static_assert(RP % 32 == 0 && RP <= 256, "rank padding must be a multiple of 32, at most 256");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);  // [kStages] TMA landed
  uint64_t* empty = full + S::kStages;                             // [kStages] MMA done with the stage
  uint64_t* aready = empty + S::kStages;                           // [2] operand written by warps 0-7
  uint64_t* afree = aready + 2;                                    // [2] MMA done reading the operand
  uint64_t* mma_done = afree + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t csize = cluster_size();
  const uint32_t crank = cluster_rank();
  const int m0 = (blockIdx.x / csize) * kRows;
  const int nchunks = p.K / kChunk;
  const int c_begin = static_cast<int>(crank * nchunks / csize);
  const int c_end = static_cast<int>((crank + 1) * nchunks / csize);
  const int nlocal = c_end - c_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&aready[b], kQWarps);
      mbar_init(&afree[b], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kQWarps) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kQWarps) {
    // ------------------------------------------------ TMA producer + MMA issuer
    if (lane == 0) {
      prefetch_tensormap(&maps.x);
      prefetch_tensormap(&maps.l1t);
      const uint32_t idesc = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kRows, RP);
      int issued = 0;
      bool ok = true;
      auto issue = [&](int j) -> bool {
        const int s = j % S::kStages;
        if (!mbar_wait(&empty[s], ((j / S::kStages) & 1) ^ 1, abort_flag, p.status)) return false;
        uint8_t* st = smem + s * S::kStage;
        mbar_arrive_expect_tx(&full[s], S::kX + S::kL + kChunk * 4);
        tma_load_2d(st, &maps.x, &full[s], (c_begin + j) * kChunk, m0);
        tma_load_2d(st + S::kX, &maps.l1t, &full[s], (c_begin + j) * kChunk, 0);
        bulk_load(st + S::kX + S::kL, p.inv_s + (c_begin + j) * kChunk, kChunk * 4, &full[s]);
        return true;
      };
      for (; issued < nlocal && issued < S::kStages - 1 && ok; ++issued) ok = issue(issued);
      for (int j = 0; j < nlocal && ok; ++j) {
        if (issued < nlocal) {
          ok = issue(issued);
          if (!ok) break;
          ++issued;
        }
        const int b = j & 1;
        ok = mbar_wait(&aready[b], (j >> 1) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const int s = j % S::kStages;
        const uint32_t a_hi = smem_u32(smem + S::kAOff + b * S::kA);
        const uint32_t a_lo = a_hi + kRows * 128;
        const uint32_t bt = smem_u32(smem + s * S::kStage + S::kX);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bd = smem_desc(bt + 32 * ks, 16, 1024, kSw128);
          mma_f16(tmem, smem_desc(a_hi + 32 * ks, 16, 1024, kSw128), bd, idesc, (j > 0 || ks > 0) ? 1u : 0u);
          mma_f16(tmem, smem_desc(a_lo + 32 * ks, 16, 1024, kSw128), bd, idesc, 1u);
        }
        tc_commit(&empty[s]);
        tc_commit(&afree[b]);
      }
      if (!ok) {
        // let the copies still in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int j = max(0, issued - S::kStages); j < issued; ++j)
          mbar_wait(&full[j % S::kStages], (j / S::kStages) & 1, &no_abort, nullptr);
      }
      tc_commit(mma_done);  // arrives once every MMA issued above has finished
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ quantizing warps
    const int cs = lane & 7;   // 16-byte column segment of the chunk
    const int rl = lane >> 3;  // row within a 4-row pass
    const int r0 = warp * (kRows / kQWarps);  // this warp's rows
    for (int j = 0; j < nlocal; ++j) {
      const int s = j % S::kStages;
      const int b = j & 1;
      if (!mbar_wait(&full[s], (j / S::kStages) & 1, abort_flag, p.status)) break;
      if (j >= 2 && !mbar_wait(&afree[b], ((j >> 1) & 1) ^ 1, abort_flag, p.status)) break;
      const uint8_t* xt = smem + s * S::kStage;
      uint8_t* ahi = smem + S::kAOff + b * S::kA;
      uint8_t* alo = ahi + kRows * 128;
      const int k = (c_begin + j) * kChunk + cs * 8;
      const float* inv_s = reinterpret_cast<const float*>(xt + S::kX + S::kL) + cs * 8;
      const float4 is0 = *reinterpret_cast<const float4*>(inv_s);
      const float4 is1 = *reinterpret_cast<const float4*>(inv_s + 4);
      const float is[8] = {is0.x, is0.y, is0.z, is0.w, is1.x, is1.y, is1.z, is1.w};
#pragma unroll
      for (int i = 0; i < kRows / kQWarps / 4; ++i) {
        const int lrow = r0 + 4 * i + rl;
        const int phys = (cs ^ (lrow & 7)) * 16;
        const uint4 xv = *reinterpret_cast<const uint4*>(xt + lrow * 128 + phys);
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // one IEEE round-to-nearest product per element (packed pair)
          const float2 pr = __fmul2_rn(make_float2(bf16_lo(w[e]), bf16_hi(w[e])), make_float2(is[2 * e], is[2 * e + 1]));
          v[2 * e] = pr.x;
          v[2 * e + 1] = pr.y;
        }
        quantize8<FMT>(v, p, m0 + lrow, k, cs);
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * e]);
          const __nv_bfloat16 h1 = __float2bfloat16_rn(v[2 * e + 1]);
          const float d0 = v[2 * e] - __bfloat162float(h0);
          const float d1 = v[2 * e + 1] - __bfloat162float(h1);
          h[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          l[e] = pack_bf16x2(d0, d1);
        }
        // same 128-byte swizzle as the TMA tiles: the canonical tcgen05 K-major layout
        *reinterpret_cast<uint4*>(ahi + lrow * 128 + phys) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(alo + lrow * 128 + phys) = make_uint4(l[0], l[1], l[2], l[3]);
      }
      fence_async_smem();  // make the generic-proxy writes visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[b]);
    }
  }

  // ------------------------------------------------ cluster reduction of T
  {
    volatile int no_abort = 0;
    mbar_wait(mma_done, 0, &no_abort, nullptr);
  }
  tc_fence_after();
  const bool healthy = !*abort_flag;
  float* red = reinterpret_cast<float*>(smem + S::kRedOff);
  const uint32_t red_s = smem_u32(red);
  for (int c0 = 0; c0 < RP; c0 += S::kRedW) {
    // 1. each CTA parks its partial [128 x kRedW] fp32 in its own shared memory
    if (warp < 8 && healthy) {
      const int q = warp & 3;
      const int half = warp >> 2;
      if (half * 32 < S::kRedW) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + c0 + half * 32, r);
        tmem_ld_wait();
        float* dst = red + (32 * q + lane) * S::kRedW + half * 32;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                            __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
      }
    }
    cluster_sync();
    // 2. CTA r sums rows [r*128/S, (r+1)*128/S) over the cluster, rank 0 first
    if (healthy) {
      const int rows_per = kRows / static_cast<int>(csize);
      const int rbeg = static_cast<int>(crank) * rows_per;
      const int nvec = rows_per * (S::kRedW / 4);
      for (int i = threadIdx.x; i < nvec; i += kThreads) {
        const int row = rbeg + i / (S::kRedW / 4);
        const int col = (i % (S::kRedW / 4)) * 4;
        const uint32_t off = static_cast<uint32_t>((row * S::kRedW + col) * 4);
        float4 part[8];
#pragma unroll
        for (uint32_t pr = 0; pr < 8; ++pr)
          if (pr < csize) part[pr] = ld_peer_v4(map_peer(red_s + off, pr));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (uint32_t pr = 0; pr < 8; ++pr)
          if (pr < csize) {  // fixed rank order: deterministic sums
            acc.x += part[pr].x;
            acc.y += part[pr].y;
            acc.z += part[pr].z;
            acc.w += part[pr].w;
          }
        const float sc = p.t_scale;
        uint2 out = make_uint2(pack_bf16x2(acc.x * sc, acc.y * sc), pack_bf16x2(acc.z * sc, acc.w * sc));
        *reinterpret_cast<uint2*>(p.T + static_cast<size_t>(m0 + row) * RP + c0 + col) = out;
      }
    }
    cluster_sync();  // peers are done reading before the buffer is reused or the CTA exits
  }

  // ------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kQWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

// Cluster size: the largest power of two <= 8 whose clusters all fit on the
// GPU at once (cluster placement, not just the SM count, decides that) and
// that leaves every CTA at least one chunk.
template <class Kern>
int choose_split(Kern kern, int smem, int row_blocks, int nchunks) {
  int best = 1;
  for (int s = 2; s <= 8 && s <= nchunks; s *= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(row_blocks * s, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = s;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      break;
    }
    if (clusters >= row_blocks) best = s;
  }
  return best;
}

template <int FMT, int RP>
cudaError_t launch_rp(const ActQuantParams& p, const ActQuantMaps& maps, cudaStream_t stream) {
  using S = K1Shape<RP>;
  auto kern = act_quant_kernel<FMT, RP>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int row_blocks = p.M_pad / kRows;
  static int cached_rb = -1, cached_k = -1, cached_split = 1;
  if (row_blocks != cached_rb || p.K != cached_k) {
    cached_split = choose_split(kern, S::kTotal, row_blocks, p.K / kChunk);
    cached_rb = row_blocks;
    cached_k = p.K;
  }
  const int split = cached_split;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(row_blocks * split, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = S::kTotal;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, maps);
}

template <int FMT>
cudaError_t launch_fmt(const ActQuantParams& p, const ActQuantMaps& maps, int rp, cudaStream_t stream) {
  switch (rp) {
    case 32: return launch_rp<FMT, 32>(p, maps, stream);
    case 64: return launch_rp<FMT, 64>(p, maps, stream);
    case 96: return launch_rp<FMT, 96>(p, maps, stream);
    case 128: return launch_rp<FMT, 128>(p, maps, stream);
    case 160: return launch_rp<FMT, 160>(p, maps, stream);
    case 192: return launch_rp<FMT, 192>(p, maps, stream);
    case 224: return launch_rp<FMT, 224>(p, maps, stream);
    case 256: return launch_rp<FMT, 256>(p, maps, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int act_quant_box_rows() { return kRows; }

cudaError_t launch_act_quant(const ActQuantParams& p, const ActQuantMaps& maps, int fmt, int rp,
                             cudaStream_t stream) {
  if (p.M_pad % 128 != 0 || p.K % 128 != 0) return cudaErrorInvalidValue;
  if (fmt == SVDQ_INT4_G64) return launch_fmt<SVDQ_INT4_G64>(p, maps, rp, stream);
  return launch_fmt<SVDQ_NVFP4_G16>(p, maps, rp, stream);
}

}  // namespace svdq
