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
// Work split: CTA (b, s) owns rows [128 b, 128 b + 128) and the s-th of S
// equal shares of K, walked in 64-column chunks. S is chosen so that the grid
// fills the GPU in one wave; the CTAs never wait on one another. Per chunk:
//   * warp 17 (one thread) streams the X tile [128 x 64], the L1^T slice
//     [RP x 64] and the inv_s slice into a shared-memory ring with TMA / bulk
//     copies (128-byte swizzle). The ring is as deep as shared memory allows
//     (7 stages at RP = 32): X comes from HBM, and the loads in flight are
//     what sets its bandwidth;
//   * warps 0-15: each thread owns 16 consecutive elements of one row (a
//     whole NVFP4 group; a quarter of an INT4 group, whose amax takes two
//     shuffles). It smooths, quantizes, stores codes and scales, and writes
//     x_hat as a bf16 high part and a bf16 remainder straight into a tcgen05
//     K-major operand buffer;
//   * one thread of warp 16 then issues tcgen05 kind::f16 MMAs
//     (M = 128, N = RP, bf16 x bf16 -> fp32) of hi and lo against L1 into a
//     TMEM accumulator, so x_hat enters the product with float accuracy.
// At the end each CTA parks its float partial product over its share of K in
// the workspace and counts itself in on its row block's arrival counter; the
// last of the S CTAs to arrive sums the S partials in share order (the same
// sum whatever the arrival order), scales by t_scale, stores T as bf16 and
// resets the counter for the next launch. With S = 1 the CTA stores T
// directly.
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

constexpr int kRows = 128;         // rows per CTA (the MMA's M)
constexpr int kQWarps = 16;        // quantizing warps, 8 rows each
constexpr int kMmaWarp = kQWarps;  // TMEM owner + MMA issuer
constexpr int kProdWarp = kQWarps + 1;
constexpr int kThreads = (kQWarps + 2) * 32;
constexpr int kChunk = 64;         // columns per chunk (one 128-byte swizzle atom of bf16)
constexpr int kMaxSplit = 16;      // K shares per row block (bounds the partials the last CTA sums)

template <int RP>
struct K1Shape {
  static constexpr int kABufs = 2;                   // x_hat operand buffers
  static constexpr int kX = kRows * 128;             // X tile of a chunk (bf16, 64 cols)
  static constexpr int kL = RP * 128;                // L1^T slice of a chunk
  static constexpr int kS = 256;                     // inv_s slice of a chunk
  static constexpr int kStage = ((kX + kL + kS + 1023) / 1024) * 1024;  // 128-byte-swizzled TMA tiles start 1 KB-aligned
  static constexpr int kAHalf = kRows * 128;         // one operand (hi or lo) of a chunk
  static constexpr int kA = 2 * kAHalf;              // hi + lo MMA operand of a chunk
  static constexpr int kBudget = 232448 - 1024 - 512;  // dynamic shared memory, less alignment slack and barriers
  static constexpr int kStagesFit = (kBudget - kABufs * kA) / kStage;
  static constexpr int kStages = kStagesFit < 8 ? kStagesFit : 8;
  static constexpr int kAOff = kStages * kStage;
  static constexpr int kBarOff = kAOff + kABufs * kA;
  static constexpr int kTotal = kBarOff + 256 + 1024;
  static_assert(kStages >= 2 && kTotal <= 232448, "shared memory budget");
  static_assert(kX % 1024 == 0 && kL % 1024 == 0, "TMA destinations stay 1024-byte aligned");
  static constexpr int kMinBlocks = 1;
  static constexpr uint32_t kTmemCols = RP <= 32 ? 32 : (RP <= 64 ? 64 : (RP <= 128 ? 128 : 256));
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Quantize this thread's 16 consecutive smoothed values v (row `row`, columns
// k0 .. k0+15) and store their codes and group scale.
template <int FMT>
__device__ __forceinline__ void quantize16(const float (&v)[16], const ActQuantParams& p, int row, int k0, int seg) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = fmaxf(m[i], m[i + 4]);
  float amax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
  if (FMT == SVDQ_INT4_G64) {
    // a group of 64 = the 4 lanes of this row (lane >> 2 shared)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float safe = amax > 0.f ? amax : 1.f;
    const float scale = amax > 0.f ? __fdiv_rn(safe, 7.0f) : 0.f;
    const float inv = __fdiv_rn(7.0f, safe);
    // |v| <= amax and inv <= (7 / amax)(1 + 2^-24), so |v * inv| rounds to at
    // most 7: rint already lands in [-7, 7] and the [-8, 7] clamp never acts.
    // An all-zero group gives v = 0 and codes 0 with the placeholder inv.
    // The rounding must see the float32-rounded product, so it is rintf on
    // the product (an add-based round-to-integer would be fused with the
    // multiply into one FMA and round the exact product instead).
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p01 = __fmul2_rn(make_float2(v[4 * i], v[4 * i + 1]), make_float2(inv, inv));
      const float2 p23 = __fmul2_rn(make_float2(v[4 * i + 2], v[4 * i + 3]), make_float2(inv, inv));
      c[i] = cvt_e4m3x2(rintf(p01.x), rintf(p01.y)) | (cvt_e4m3x2(rintf(p23.x), rintf(p23.y)) << 16);
    }
    *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * p.K + k0) = make_uint4(c[0], c[1], c[2], c[3]);
    if (seg == 0) reinterpret_cast<float*>(p.scales)[static_cast<size_t>(k0 >> 6) * p.M_pad + row] = scale;
  } else {
    // a group of 16 = this thread's values
    const uint32_t sb = cvt_e4m3x2(__fdiv_rn(amax, p.denom), 0.f) & 0xFFu;
    const float eff = __fmul_rn(e4m3_to_float(sb), p.g_x);
    const float inv = __frcp_rn(eff != 0.f ? eff : 1.f);
    float q[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 pr = __fmul2_rn(make_float2(v[8 * h + j], v[8 * h + j + 1]), make_float2(inv, inv));
        q[h][j] = pr.x;
        q[h][j + 1] = pr.y;
      }
    const uint32_t c0 = eff != 0.f ? cvt_e2m1x8(q[0]) : 0u;
    const uint32_t c1 = eff != 0.f ? cvt_e2m1x8(q[1]) : 0u;
    *reinterpret_cast<uint2*>(p.codes + static_cast<size_t>(row) * (p.K >> 1) + (k0 >> 1)) = make_uint2(c0, c1);
    // scale-factor atom: (row / 128) * (K / 64) + k / 64, byte (row % 32) * 16 + ((row / 32) % 4) * 4 + (k / 16) % 4
    const size_t atom = static_cast<size_t>(row >> 7) * (p.K >> 6) + (k0 >> 6);
    const int off = (row & 31) * 16 + ((row >> 5) & 3) * 4 + ((k0 >> 4) & 3);
    reinterpret_cast<uint8_t*>(p.scales)[atom * 512 + off] = static_cast<uint8_t>(sb);
  }
}

template <int FMT, int RP>
__global__ void __launch_bounds__(kThreads, K1Shape<RP>::kMinBlocks)
    act_quant_kernel(const ActQuantParams p, const __grid_constant__ ActQuantMaps maps) {
  using S = K1Shape<RP>;
  static_assert(RP % 32 == 0 && RP <= 256, "rank padding must be a multiple of 32, at most 256");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);  // [kStages] TMA landed
  uint64_t* empty = full + S::kStages;                             // [kStages] MMA done with the stage
  uint64_t* aready = empty + S::kStages;                           // [kABufs] operand written by warps 0-15
  uint64_t* afree = aready + S::kABufs;                            // [kABufs] MMA done reading the operand
  uint64_t* mma_done = afree + S::kABufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* is_last = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = p.split;
  const int rb = blockIdx.x / split;
  const int sh = blockIdx.x % split;  // this CTA's share of K
  const int m0 = rb * kRows;
  const int nchunks = p.K / kChunk;
  const int c_begin = sh * nchunks / split;
  const int c_end = (sh + 1) * nchunks / split;
  const int nlocal = c_end - c_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < S::kABufs; ++b) {
      mbar_init(&aready[b], kQWarps);
      mbar_init(&afree[b], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProdWarp) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&maps.x);
      prefetch_tensormap(&maps.l1t);
      int j = 0;
      for (; j < nlocal; ++j) {
        const int s = j % S::kStages;
        if (!mbar_wait(&empty[s], ((j / S::kStages) & 1) ^ 1, abort_flag, p.status)) break;
        uint8_t* st = smem + s * S::kStage;
        mbar_arrive_expect_tx(&full[s], S::kX + S::kL + kChunk * 4);
        tma_load_2d(st, &maps.x, &full[s], (c_begin + j) * kChunk, m0);
        tma_load_2d(st + S::kX, &maps.l1t, &full[s], (c_begin + j) * kChunk, 0);
        bulk_load(st + S::kX + S::kL, p.inv_s + (c_begin + j) * kChunk, kChunk * 4, &full[s]);
      }
      if (j < nlocal) {
        // gave up: let the copies still in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int i = max(0, j - S::kStages); i < j; ++i)
          mbar_wait(&full[i % S::kStages], (i / S::kStages) & 1, &no_abort, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kRows, RP);
      for (int j = 0; j < nlocal; ++j) {
        const int b = j % S::kABufs;
        if (!mbar_wait(&aready[b], (j / S::kABufs) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const int s = j % S::kStages;
        const uint32_t a_hi = smem_u32(smem + S::kAOff + b * S::kA);
        const uint32_t a_lo = a_hi + S::kAHalf;
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
      tc_commit(mma_done);  // arrives once every MMA issued above has finished
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ quantizing warps
    const int seg = lane & 3;                 // 16-column segment of the chunk
    const int lrow = warp * 8 + (lane >> 2);  // row within the CTA
    const int row = m0 + lrow;
    for (int j = 0; j < nlocal; ++j) {
      const int s = j % S::kStages;
      const int b = j % S::kABufs;
      if (!mbar_wait(&full[s], (j / S::kStages) & 1, abort_flag, p.status)) break;
      if (j >= S::kABufs && !mbar_wait(&afree[b], ((j / S::kABufs) & 1) ^ 1, abort_flag, p.status)) break;
      const uint8_t* xt = smem + s * S::kStage;
      const float4* is4 = reinterpret_cast<const float4*>(xt + S::kX + S::kL) + 4 * seg;
      const uint32_t phys0 = lrow * 128 + (((2 * seg) ^ (lrow & 7)) * 16);
      const uint32_t phys1 = lrow * 128 + (((2 * seg + 1) ^ (lrow & 7)) * 16);
      const uint4 x0 = *reinterpret_cast<const uint4*>(xt + phys0);
      const uint4 x1 = *reinterpret_cast<const uint4*>(xt + phys1);
      const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      float v[16];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 is = is4[e];
        // one IEEE round-to-nearest product per element (packed pairs)
        const float2 a = __fmul2_rn(make_float2(bf16_lo(w[2 * e]), bf16_hi(w[2 * e])), make_float2(is.x, is.y));
        const float2 c = __fmul2_rn(make_float2(bf16_lo(w[2 * e + 1]), bf16_hi(w[2 * e + 1])), make_float2(is.z, is.w));
        v[4 * e] = a.x;
        v[4 * e + 1] = a.y;
        v[4 * e + 2] = c.x;
        v[4 * e + 3] = c.y;
      }
      quantize16<FMT>(v, p, row, (c_begin + j) * kChunk + 16 * seg, seg);
      // x_hat = hi + lo with hi = bf16(x_hat) and lo = bf16(x_hat - hi) (the
      // difference is exact in float), in the same 128-byte swizzle as the
      // TMA tiles: the canonical tcgen05 K-major layout
      uint32_t h[8], l[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        const float2 d = __fadd2_rn(make_float2(v[2 * e], v[2 * e + 1]), make_float2(-bf16_lo(h[e]), -bf16_hi(h[e])));
        l[e] = pack_bf16x2(d.x, d.y);
      }
      uint8_t* ad = smem + S::kAOff + b * S::kA;
      *reinterpret_cast<uint4*>(ad + phys0) = make_uint4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint4*>(ad + phys1) = make_uint4(h[4], h[5], h[6], h[7]);
      *reinterpret_cast<uint4*>(ad + S::kAHalf + phys0) = make_uint4(l[0], l[1], l[2], l[3]);
      *reinterpret_cast<uint4*>(ad + S::kAHalf + phys1) = make_uint4(l[4], l[5], l[6], l[7]);
      fence_async_smem();  // make the generic-proxy writes visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[b]);
    }
  }

  // ------------------------------------------------ this CTA's share of T
  {
    volatile int no_abort = 0;
    mbar_wait(mma_done, 0, &no_abort, nullptr);
  }
  tc_fence_after();
  const bool healthy = !*abort_flag;
  // warp q may read TMEM lanes 32q .. 32q+31: rows 32q .. 32q+31 of the CTA
  const int r = m0 + 32 * warp + lane;
  const float sc = p.t_scale;
  if (split == 1) {
    if (warp < 4 && healthy) {
#pragma unroll 1
      for (int c0 = 0; c0 < RP; c0 += 32) {
        uint32_t acc[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, acc);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          const uint4 o = make_uint4(
              pack_bf16x2(__uint_as_float(acc[e]) * sc, __uint_as_float(acc[e + 1]) * sc),
              pack_bf16x2(__uint_as_float(acc[e + 2]) * sc, __uint_as_float(acc[e + 3]) * sc),
              pack_bf16x2(__uint_as_float(acc[e + 4]) * sc, __uint_as_float(acc[e + 5]) * sc),
              pack_bf16x2(__uint_as_float(acc[e + 6]) * sc, __uint_as_float(acc[e + 7]) * sc));
          *reinterpret_cast<uint4*>(p.T + static_cast<size_t>(r) * RP + c0 + e) = o;
        }
      }
    }
  } else {
    if (warp < 4) {
      // park this share's partial; a CTA that gave up parks zeros, so the
      // arrival count stays right and the status word reports the failure
      float* dst = p.Tpart + (static_cast<size_t>(sh) * p.M_pad + r) * RP;
#pragma unroll 1
      for (int c0 = 0; c0 < RP; c0 += 32) {
        uint32_t acc[32];
        if (healthy) {
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, acc);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + c0 + e) = make_float4(__uint_as_float(acc[e]), __uint_as_float(acc[e + 1]),
                                                                 __uint_as_float(acc[e + 2]), __uint_as_float(acc[e + 3]));
      }
      __threadfence();  // the partial is visible device-wide before this CTA counts itself in
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const int prev = atomicAdd(p.counters + rb, 1);
      const int last = prev == split - 1;
      if (last) p.counters[rb] = 0;  // every share has arrived: ready for the next launch
      *is_last = last;
    }
    __syncthreads();
    if (*is_last && warp < kQWarps) {
      __threadfence();  // acquire side: the other shares' partials are visible
      // all quantizing threads sum: one 8-column slice of one row per item,
      // four shares' loads in flight at a time, shares added in order
      constexpr int kSlices = RP / 8;
#pragma unroll 1
      for (int item = threadIdx.x; item < kRows * kSlices; item += kQWarps * 32) {
        const int rr = m0 + item / kSlices;
        const int c0 = (item % kSlices) * 8;
        const float* src = p.Tpart + static_cast<size_t>(rr) * RP + c0;
        const size_t stride = static_cast<size_t>(p.M_pad) * RP;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int t0 = 0; t0 < split; t0 += 4) {
          float4 u[4], w[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (t0 + t < split) {
              u[t] = __ldcg(reinterpret_cast<const float4*>(src + (t0 + t) * stride));
              w[t] = __ldcg(reinterpret_cast<const float4*>(src + (t0 + t) * stride + 4));
            }
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (t0 + t < split) {  // share order: the same sum whatever the arrival order
              acc[0] += u[t].x; acc[1] += u[t].y; acc[2] += u[t].z; acc[3] += u[t].w;
              acc[4] += w[t].x; acc[5] += w[t].y; acc[6] += w[t].z; acc[7] += w[t].w;
            }
          }
        }
        const uint4 o = make_uint4(pack_bf16x2(acc[0] * sc, acc[1] * sc), pack_bf16x2(acc[2] * sc, acc[3] * sc),
                                   pack_bf16x2(acc[4] * sc, acc[5] * sc), pack_bf16x2(acc[6] * sc, acc[7] * sc));
        *reinterpret_cast<uint4*>(p.T + static_cast<size_t>(rr) * RP + c0) = o;
      }
    }
  }

  // ------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

template <int FMT, int RP>
cudaError_t launch_rp(const ActQuantParams& p, const ActQuantMaps& maps, cudaStream_t stream) {
  using S = K1Shape<RP>;
  auto kern = act_quant_kernel<FMT, RP>;
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
  });
  if (e != cudaSuccess) return e;
  act_quant_kernel<FMT, RP><<<(p.M_pad / kRows) * p.split, kThreads, S::kTotal, stream>>>(p, maps);
  return cudaGetLastError();
}

template <int FMT, int RP>
int resident_ctas() {
  using S = K1Shape<RP>;
  auto kern = act_quant_kernel<FMT, RP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal) != cudaSuccess) return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, S::kTotal) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 1;
  }
  return n;
}

template <int FMT>
int resident_fmt(int rp) {
  switch (rp) {
    case 32: return resident_ctas<FMT, 32>();
    case 64: return resident_ctas<FMT, 64>();
    case 96: return resident_ctas<FMT, 96>();
    case 128: return resident_ctas<FMT, 128>();
    case 160: return resident_ctas<FMT, 160>();
    case 192: return resident_ctas<FMT, 192>();
    case 224: return resident_ctas<FMT, 224>();
    case 256: return resident_ctas<FMT, 256>();
    default: return 1;
  }
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

int act_quant_split(int M_pad, int K, int fmt, int rp, int sms) {
  // CTAs that fit on the GPU at once, divided among the 64-row blocks; each
  // CTA keeps at least one chunk, and at most kMaxSplit partials are summed.
  // resident CTAs per SM for (format, rank padding), queried once per process
  static int cache[2][9] = {};
  const int fi = fmt == SVDQ_INT4_G64 ? 0 : 1, ri = rp / 32;
  if (ri < 1 || ri > 8) return 1;
  if (cache[fi][ri] == 0)
    cache[fi][ri] = fmt == SVDQ_INT4_G64 ? resident_fmt<SVDQ_INT4_G64>(rp) : resident_fmt<SVDQ_NVFP4_G16>(rp);
  const int per_sm = cache[fi][ri];
  const int row_blocks = M_pad / kRows;
  int split = (sms * per_sm) / row_blocks;
  const int nchunks = K / kChunk;
  if (split > nchunks) split = nchunks;
  if (split > kMaxSplit) split = kMaxSplit;
  return split < 1 ? 1 : split;
}

cudaError_t launch_act_quant(const ActQuantParams& p, const ActQuantMaps& maps, int fmt, int rp,
                             cudaStream_t stream) {
  if (p.M_pad % 128 != 0 || p.K % 128 != 0 || p.split < 1 || p.M_pad / kRows > kMaxRowBlocks ||
      (p.split > 1 && (!p.Tpart || !p.counters)))
    return cudaErrorInvalidValue;
  if (fmt == SVDQ_INT4_G64) return launch_fmt<SVDQ_INT4_G64>(p, maps, rp, stream);
  return launch_fmt<SVDQ_NVFP4_G16>(p, maps, rp, stream);
}

}  // namespace svdq
