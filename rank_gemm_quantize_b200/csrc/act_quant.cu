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
// The branch input is computed as T = X (diag(s)^-1 L1): the layer keeps the
// factor L1s = fp32(inv_s[k] L1[k, j]) as a bf16 pair hi + lo (hi = bf16(L1s),
// lo = bf16(L1s - hi), about 16 significant bits together), so the tensor core
// reads the bf16 X tile exactly as TMA brought it in and
// T = X L1s_hi + X L1s_lo, an associative regrouping of X diag(s)^-1 L1.
// The quantizers never have to build an MMA operand.
//
// Work split: CTA (b, s) owns rows [128 b, 128 b + 128) and the s-th of S
// equal shares of K, walked in 64-column chunks. S is chosen so that the grid
// fills the GPU in one wave; the CTAs never wait on one another. Per chunk:
//   * warp 17 (one thread) streams the X tile [128 x 64], the two L1s^T
//     slices [RP x 64] and the inv_s slice into a shared-memory ring with TMA
//     and bulk copies (128-byte swizzle). The ring is as deep as shared memory
//     allows (8 stages at RP = 32): X comes from HBM, and the bytes in flight
//     set its bandwidth;
//   * one thread of warp 16 issues the tcgen05 kind::f16 MMAs
//     (M = 128, N = RP, bf16 x bf16 -> fp32) of the X tile against hi and lo
//     into a TMEM accumulator;
//   * warps 0-15: each thread owns 16 consecutive elements of one row, two
//     chunks at a time for independent work (a whole NVFP4 group; a quarter
//     of an INT4 group, whose amax takes two shuffles). It smooths,
//     quantizes and stores codes and scales.
// A stage is free again once the MMAs that read it have completed and all 16
// quantizing warps have read it.
// At the end each CTA parks its float partial product over its share of K in
// the workspace and counts itself in on its row block's arrival counter; the
// last of the S CTAs to arrive sums the S partials in share order (the same
// sum whatever the arrival order), scales by t_scale, stores T as bf16 and
// resets the counter for the next launch. With S = 1 the CTA stores T
// directly. T columns that belong to a LoRA adapter a row has not selected
// (per-row adapter mask) are stored as zero. RP = 0 (no branch: the
// smoothing-only special case) compiles without TMEM, MMAs or T.
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
  static constexpr int kX = kRows * 128;             // X tile of a chunk (bf16, 64 cols)
  static constexpr int kL = RP * 128;                // one L1s^T slice (hi or lo) of a chunk
  static constexpr int kS = 256;                     // inv_s slice of a chunk
  static constexpr int kStage = ((kX + 2 * kL + kS + 1023) / 1024) * 1024;  // swizzled TMA tiles start 1 KB-aligned
  static constexpr int kBudget = 232448 - 1024 - 512;  // dynamic shared memory, less alignment slack and barriers
  static constexpr int kStagesFit = kBudget / kStage;
  static constexpr int kStages = kStagesFit < 8 ? kStagesFit : 8;
  static constexpr int kBarOff = kStages * kStage;
  static constexpr int kTotal = kBarOff + 256 + 1024;
  static_assert(kStages >= 2 && kTotal <= 232448, "shared memory budget");
  static_assert(kX % 1024 == 0 && kL % 1024 == 0, "TMA destinations stay 1024-byte aligned");
  static constexpr uint32_t kTmemCols = RP <= 32 ? 32 : (RP <= 64 ? 64 : (RP <= 128 ? 128 : 256));
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Quantize this thread's 16 consecutive smoothed values v (row `row`, columns
// k0 .. k0+15) and store their codes and group scale.
template <int FMT>
__device__ __forceinline__ void quantize16(const float (&v)[16], const ActQuantParams& p, int row, int k0, int seg) {
  if (FMT == SVDQ_INT4_G64) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = fmaxf(m[i], m[i + 4]);
    float amax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
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
    uint32_t c0, c1;
    const uint32_t sb = nvfp4_quant16(v, p.denom, p.g_x, c0, c1);
    *reinterpret_cast<uint2*>(p.codes + static_cast<size_t>(row) * (p.K >> 1) + (k0 >> 1)) = make_uint2(c0, c1);
    // scale-factor atom: (row / 128) * (K / 64) + k / 64, byte (row % 32) * 16 + ((row / 32) % 4) * 4 + (k / 16) % 4
    const size_t atom = static_cast<size_t>(row >> 7) * (p.K >> 6) + (k0 >> 6);
    const int off = (row & 31) * 16 + ((row >> 5) & 3) * 4 + ((k0 >> 4) & 3);
    reinterpret_cast<uint8_t*>(p.scales)[atom * 512 + off] = static_cast<uint8_t>(sb);
  }
}

// This thread's 16 smoothed values of one chunk: x_hat = fp32(x * inv_s),
// one IEEE round-to-nearest product per element (packed pairs).
__device__ __forceinline__ void smooth16(const uint8_t* xt, const float4* is4, uint32_t phys0, uint32_t phys1,
                                         float (&v)[16]) {
  const uint4 x0 = *reinterpret_cast<const uint4*>(xt + phys0);
  const uint4 x1 = *reinterpret_cast<const uint4*>(xt + phys1);
  const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 is = is4[e];
    const float2 a = __fmul2_rn(make_float2(bf16_lo(w[2 * e]), bf16_hi(w[2 * e])), make_float2(is.x, is.y));
    const float2 c = __fmul2_rn(make_float2(bf16_lo(w[2 * e + 1]), bf16_hi(w[2 * e + 1])), make_float2(is.z, is.w));
    v[4 * e] = a.x;
    v[4 * e + 1] = a.y;
    v[4 * e + 2] = c.x;
    v[4 * e + 3] = c.y;
  }
}

// Whether branch column c of row `mask` is kept: the base factor's columns
// always; an adapter's columns when the row selected its slot.
__device__ __forceinline__ bool column_on(const ActQuantParams& p, uint32_t mask, int c) {
  if (c < p.col_start[0]) return true;
#pragma unroll
  for (int s = 0; s < kMaxAdapters; ++s)
    if (c < p.col_start[s + 1]) return (mask >> s) & 1u;
  return true;  // padding columns (always zero)
}

// Stores 8 consecutive T columns c0 .. c0+7 of row r (scaled by t_scale, the
// columns of unselected adapters zeroed); with T_lo also the bf16 remainders.
__device__ __forceinline__ void store_t8(const ActQuantParams& p, int RP, int r, int c0, const float (&a)[8]) {
  float v[8];
  // the mask has one entry per row of X; padding rows (r >= M) hold zeros anyway
  const bool masked = p.row_mask != nullptr && r < p.M;
  const uint32_t mask = masked ? __ldg(p.row_mask + r) : 0xFFFFFFFFu;
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = (masked && !column_on(p, mask, c0 + e)) ? 0.f : a[e] * p.t_scale;
  const uint4 o = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                             pack_bf16x2(v[6], v[7]));
  const size_t off = static_cast<size_t>(r) * RP + c0;
  *reinterpret_cast<uint4*>(p.T + off) = o;
  if (p.T_lo) {
    const uint32_t w[4] = {o.x, o.y, o.z, o.w};
    uint32_t l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      l[e] = pack_bf16x2(v[2 * e] - __uint_as_float(w[e] << 16), v[2 * e + 1] - __uint_as_float(w[e] & 0xFFFF0000u));
    *reinterpret_cast<uint4*>(p.T_lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

template <int FMT, int RP>
__global__ void __launch_bounds__(kThreads, 1)
    act_quant_kernel(const ActQuantParams p, const __grid_constant__ ActQuantMaps maps) {
  using S = K1Shape<RP>;
  constexpr bool kBranch = RP > 0;
  static_assert(RP % 32 == 0 && RP <= 256, "rank padding must be a multiple of 32, at most 256");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);  // [kStages] TMA landed
  uint64_t* empty = full + S::kStages;                             // [kStages] MMAs and quantizers done with it
  uint64_t* mma_done = empty + S::kStages;
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
      mbar_init(&empty[s], kQWarps + (kBranch ? 1 : 0));
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (kBranch && warp == kMmaWarp) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = kBranch ? *tmem_slot : 0u;

  if (warp == kProdWarp) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&maps.x);
      if (kBranch) {
        prefetch_tensormap(&maps.l1h);
        prefetch_tensormap(&maps.l1l);
      }
      int j = 0;
      for (; j < nlocal; ++j) {
        const int s = j % S::kStages;
        if (!mbar_wait(&empty[s], ((j / S::kStages) & 1) ^ 1, abort_flag, p.status)) break;
        uint8_t* st = smem + s * S::kStage;
        const int kx = (c_begin + j) * kChunk;
        mbar_arrive_expect_tx(&full[s], S::kX + 2 * S::kL + kChunk * 4);
        tma_load_2d(st, &maps.x, &full[s], kx, m0);
        if (kBranch) {
          tma_load_2d(st + S::kX, &maps.l1h, &full[s], kx, 0);
          tma_load_2d(st + S::kX + S::kL, &maps.l1l, &full[s], kx, 0);
        }
        bulk_load(st + S::kX + 2 * S::kL, p.inv_s + kx, kChunk * 4, &full[s]);
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
    if (kBranch && lane == 0) {
      const uint32_t idesc = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kRows, RP > 0 ? RP : 32);
      for (int j = 0; j < nlocal; ++j) {
        const int s = j % S::kStages;
        if (!mbar_wait(&full[s], (j / S::kStages) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + s * S::kStage);
        const uint32_t bh = xa + S::kX;
        const uint32_t bl = bh + S::kL;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = smem_desc(xa + 32 * ks, 16, 1024, kSw128);
          mma_f16(tmem, ad, smem_desc(bh + 32 * ks, 16, 1024, kSw128), idesc, (j > 0 || ks > 0) ? 1u : 0u);
          mma_f16(tmem, ad, smem_desc(bl + 32 * ks, 16, 1024, kSw128), idesc, 1u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(mma_done);  // arrives once every MMA issued above has finished
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ quantizing warps
    const int seg = lane & 3;                 // 16-column segment of the chunk
    const int lrow = warp * 8 + (lane >> 2);  // row within the CTA
    const int row = m0 + lrow;
    const uint32_t phys0 = lrow * 128 + (((2 * seg) ^ (lrow & 7)) * 16);
    const uint32_t phys1 = lrow * 128 + (((2 * seg + 1) ^ (lrow & 7)) * 16);
    constexpr int kIsOff = S::kX + 2 * S::kL;
    int j = 0;
    // two chunks per pass: two independent dependency chains per thread
    for (; j + 1 < nlocal; j += 2) {
      const int s0 = j % S::kStages, s1 = (j + 1) % S::kStages;
      if (!mbar_wait(&full[s0], (j / S::kStages) & 1, abort_flag, p.status)) break;
      if (!mbar_wait(&full[s1], ((j + 1) / S::kStages) & 1, abort_flag, p.status)) break;
      const uint8_t* x0 = smem + s0 * S::kStage;
      const uint8_t* x1 = smem + s1 * S::kStage;
      float v0[16], v1[16];
      smooth16(x0, reinterpret_cast<const float4*>(x0 + kIsOff) + 4 * seg, phys0, phys1, v0);
      smooth16(x1, reinterpret_cast<const float4*>(x1 + kIsOff) + 4 * seg, phys0, phys1, v1);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s0]);
        mbar_arrive(&empty[s1]);
      }
      quantize16<FMT>(v0, p, row, (c_begin + j) * kChunk + 16 * seg, seg);
      quantize16<FMT>(v1, p, row, (c_begin + j + 1) * kChunk + 16 * seg, seg);
    }
    if (j < nlocal) {
      const int s0 = j % S::kStages;
      if (mbar_wait(&full[s0], (j / S::kStages) & 1, abort_flag, p.status)) {
        const uint8_t* x0 = smem + s0 * S::kStage;
        float v0[16];
        smooth16(x0, reinterpret_cast<const float4*>(x0 + kIsOff) + 4 * seg, phys0, phys1, v0);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s0]);
        quantize16<FMT>(v0, p, row, (c_begin + j) * kChunk + 16 * seg, seg);
      }
    }
  }

  if (kBranch) {
    // ---------------------------------------------- this CTA's share of T
    {
      volatile int no_abort = 0;
      mbar_wait(mma_done, 0, &no_abort, nullptr);
    }
    tc_fence_after();
    const bool healthy = !*abort_flag;
    // warp q may read TMEM lanes 32q .. 32q+31: rows 32q .. 32q+31 of the CTA
    const int r = m0 + 32 * warp + lane;
    if (split == 1) {
      if (warp < 4 && healthy) {
#pragma unroll 1
        for (int c0 = 0; c0 < RP; c0 += 32) {
          uint32_t acc[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, acc);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(acc[e + i]);
            store_t8(p, RP, r, c0 + e, a);
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
          store_t8(p, RP, rr, c0, acc);
        }
      }
    }
  }

  // ------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (kBranch && warp == kMmaWarp) {
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
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, S::kTotal) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 1;
  }
  return n;
}

#define SVDQ_RP_CASES(F) F(0) F(32) F(64) F(96) F(128) F(160) F(192) F(224) F(256)

template <int FMT>
int resident_fmt(int rp) {
  switch (rp) {
#define SVDQ_CASE(R) \
  case R:            \
    return resident_ctas<FMT, R>();
    SVDQ_RP_CASES(SVDQ_CASE)
#undef SVDQ_CASE
    default: return 1;
  }
}

template <int FMT>
cudaError_t launch_fmt(const ActQuantParams& p, const ActQuantMaps& maps, int rp, cudaStream_t stream) {
  switch (rp) {
#define SVDQ_CASE(R) \
  case R:            \
    return launch_rp<FMT, R>(p, maps, stream);
    SVDQ_RP_CASES(SVDQ_CASE)
#undef SVDQ_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int act_quant_box_rows() { return kRows; }

int act_quant_resident(int fmt, int rp) {
  return fmt == SVDQ_INT4_G64 ? resident_fmt<SVDQ_INT4_G64>(rp) : resident_fmt<SVDQ_NVFP4_G16>(rp);
}

int act_quant_split(int M_pad, int K, int per_sm, int sms) {
  // CTAs that fit on the GPU at once, divided among the 128-row blocks; each
  // CTA keeps at least one chunk, and at most kMaxSplit partials are summed.
  const int row_blocks = M_pad / kRows;
  int split = (sms * (per_sm < 1 ? 1 : per_sm)) / row_blocks;
  const int nchunks = K / kChunk;
  if (split > nchunks) split = nchunks;
  if (split > kMaxSplit) split = kMaxSplit;
  return split < 1 ? 1 : split;
}

cudaError_t launch_act_quant(const ActQuantParams& p, const ActQuantMaps& maps, int fmt, int rp,
                             cudaStream_t stream) {
  if (p.M_pad % 128 != 0 || p.K % 128 != 0 || p.split < 1 || p.M_pad / kRows > kMaxRowBlocks ||
      (rp > 0 && p.split > 1 && (!p.Tpart || !p.counters)) || (rp > 0 && !p.T))
    return cudaErrorInvalidValue;
  if (fmt == SVDQ_INT4_G64) return launch_fmt<SVDQ_INT4_G64>(p, maps, rp, stream);
  return launch_fmt<SVDQ_NVFP4_G16>(p, maps, rp, stream);
}

}  // namespace svdq
