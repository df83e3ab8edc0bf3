// K1: activation smoothing + 4-bit group quantization + low-rank down-projection.
//
// SVDQuant ("SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit
// Diffusion Models", abstract; msModelSlim SVDQuant entry, section 2.3, the
// dual-path output equation) runs, per layer and per input row x:
//   x_hat = x diag(s)^-1                      (the migration identity, eq. 1)
//   Q(x_hat): 4-bit codes + one scale per group along K
//   T     = x_hat L1                          (the branch input X diag(s)^-1 V)
// This kernel reads every X element once (128-bit loads), and produces all
// three in the same pass. The down-projection runs on the tensor cores
// (mma.sync bf16, fp32 accumulate) with x_hat split into a bf16 high part and
// a bf16 remainder, so T carries float32-level accuracy before its final
// rounding to bf16.
//
// Tiling: a CTA owns 32 rows and walks K in rounds of 8 chunks of 64 columns,
// one chunk per warp. Phase A (per warp): load 32x64 bf16, smooth, quantize,
// store codes/scales, stage x_hat hi/lo in shared memory. Phase B (all warps):
// the 32 x RP block of T is split into 16x8 MMA tiles, each warp accumulating
// its tiles over the round's 8 chunks. The next round's X is loaded into
// registers before phase B, so HBM reads overlap the MMAs.
//
// Numerics match the CPU oracle operation by operation: every product and
// quotient of the quantizer is a single IEEE round-to-nearest operation
// (__fmul_rn / __fdiv_rn, no FMA contraction), rint is round-half-even, and the
// E4M3 / E2M1 encodings use the hardware cvt.rn.satfinite conversions.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kRows = 32;          // rows per CTA
constexpr int kWarps = 8;          // one 64-column chunk per warp per round
constexpr int kChunk = 64;         // columns per chunk
constexpr int kSlotBytes = 2 * kRows * kChunk * 2;  // hi + lo bf16 tiles

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Quantize 8 consecutive smoothed values of one row (this lane's share of a
// group) and store the codes; returns nothing, writes the group scale from one
// lane per group.
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
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        int qi = __float2int_rn(__fmul_rn(v[j], inv));
        qi = min(7, max(-8, qi));
        q[j] = static_cast<float>(qi);
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
      for (int j = 0; j < 8; ++j) q[j] = __fmul_rn(v[j], inv);
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
__global__ void __launch_bounds__(kWarps * 32, 1) act_quant_kernel(const ActQuantParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  // 2 x (RP/8) MMA tiles of 16x8 over 8 warps: RP/32 per warp
  constexpr int kPerWarp = RP / 32;
  static_assert(RP % 32 == 0, "rank padding must be a multiple of 32");

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int m0 = blockIdx.x * kRows;
  const int cs = lane & 7;        // 16-byte column segment within a chunk
  const int rb = lane >> 3;       // row base; rows rb + 4 i
  const int nchunks = p.K / kChunk;
  const int nrounds = (nchunks + kWarps - 1) / kWarps;

  float acc[kPerWarp][4];
#pragma unroll
  for (int t = 0; t < kPerWarp; ++t)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[t][j] = 0.f;

  uint4 xr[8];
  auto load_chunk = [&](int round) {
    const int c = round * kWarps + warp;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = m0 + rb + 4 * i;
      if (c < nchunks && row < p.M) {
        xr[i] = __ldcs(reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(row) * p.K + c * kChunk + cs * 8));
      } else {
        xr[i] = make_uint4(0, 0, 0, 0);
      }
    }
  };

  load_chunk(0);
  for (int round = 0; round < nrounds; ++round) {
    // ---------------- phase A: smooth, quantize, stage hi/lo
    const int c = round * kWarps + warp;
    if (c < nchunks) {
      const int k = c * kChunk + cs * 8;
      const float4 is0 = __ldg(reinterpret_cast<const float4*>(p.inv_s + k));
      const float4 is1 = __ldg(reinterpret_cast<const float4*>(p.inv_s + k + 4));
      const float is[8] = {is0.x, is0.y, is0.z, is0.w, is1.x, is1.y, is1.z, is1.w};
      uint8_t* slot = smem + warp * kSlotBytes;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int lrow = rb + 4 * i;
        const uint32_t w[4] = {xr[i].x, xr[i].y, xr[i].z, xr[i].w};
        float v[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[2 * j] = __fmul_rn(bf16_lo(w[j]), is[2 * j]);
          v[2 * j + 1] = __fmul_rn(bf16_hi(w[j]), is[2 * j + 1]);
        }
        quantize8<FMT>(v, p, m0 + lrow, k, cs);
        uint32_t h[4], l[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * j]);
          const __nv_bfloat16 h1 = __float2bfloat16_rn(v[2 * j + 1]);
          const float r0 = v[2 * j] - __bfloat162float(h0);
          const float r1 = v[2 * j + 1] - __bfloat162float(h1);
          h[j] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                 (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          l[j] = pack_bf16x2(r0, r1);
        }
        const int phys = cs ^ (lrow & 7);
        *reinterpret_cast<uint4*>(slot + lrow * 128 + phys * 16) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(slot + kRows * 128 + lrow * 128 + phys * 16) = make_uint4(l[0], l[1], l[2], l[3]);
      }
    }
    if (round + 1 < nrounds) load_chunk(round + 1);
    __syncthreads();

    // ---------------- phase B: T += x_hat L1 over this round's chunks.
    // Warp w owns the 16-row tile mt = w & 1 and the 8-column tiles
    // nt = (w >> 1) + 4 t, so one pair of A fragments (hi, lo) feeds all of
    // its MMAs for a k-step.
    {
      const int g = lane >> 2, t4 = lane & 3;
      const int mt = warp & 1;
      const int mi = lane >> 3;
      const int arow = mt * 16 + (mi & 1) * 8 + (lane & 7);
      for (int s = 0; s < kWarps; ++s) {
        const int cc = round * kWarps + s;
        if (cc >= nchunks) break;
        const uint32_t slot = smem_u32(smem + s * kSlotBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const int kc = ks * 2 + (mi >> 1);
          const uint32_t off = arow * 128 + ((kc ^ (arow & 7)) * 16);
          uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
          ldmatrix_x4(slot + off, h0, h1, h2, h3);
          ldmatrix_x4(slot + kRows * 128 + off, l0, l1, l2, l3);
          const int k = cc * kChunk + ks * 16 + 2 * t4;
#pragma unroll
          for (int t = 0; t < kPerWarp; ++t) {
            const int nt = (warp >> 1) + 4 * t;
            const __nv_bfloat16* l1row = p.L1T + static_cast<size_t>(nt * 8 + g) * p.K;
            const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(l1row + k));
            const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(l1row + k + 8));
            mma_bf16_16816(acc[t], h0, h1, h2, h3, b0, b1);
            mma_bf16_16816(acc[t], l0, l1, l2, l3, b0, b1);
          }
        }
      }
    }
    __syncthreads();
  }

  // ---------------- write T (bf16, scaled by t_scale)
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int t = 0; t < kPerWarp; ++t) {
    const int mt = warp & 1, nt = (warp >> 1) + 4 * t;
    const int row = m0 + mt * 16 + g;
    const int col = nt * 8 + 2 * t4;
    const float sc = p.t_scale;
    *reinterpret_cast<uint32_t*>(p.T + static_cast<size_t>(row) * RP + col) =
        pack_bf16x2(acc[t][0] * sc, acc[t][1] * sc);
    *reinterpret_cast<uint32_t*>(p.T + static_cast<size_t>(row + 8) * RP + col) =
        pack_bf16x2(acc[t][2] * sc, acc[t][3] * sc);
  }
}

template <int FMT, int RP>
cudaError_t launch_rp(const ActQuantParams& p, cudaStream_t stream) {
  auto kern = act_quant_kernel<FMT, RP>;
  const int smem = kWarps * kSlotBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = p.M_pad / kRows;
  kern<<<grid, kWarps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const ActQuantParams& p, int rp, cudaStream_t stream) {
  switch (rp) {
    case 32: return launch_rp<FMT, 32>(p, stream);
    case 64: return launch_rp<FMT, 64>(p, stream);
    case 96: return launch_rp<FMT, 96>(p, stream);
    case 128: return launch_rp<FMT, 128>(p, stream);
    case 160: return launch_rp<FMT, 160>(p, stream);
    case 192: return launch_rp<FMT, 192>(p, stream);
    case 224: return launch_rp<FMT, 224>(p, stream);
    case 256: return launch_rp<FMT, 256>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_act_quant(const ActQuantParams& p, int fmt, int rp, cudaStream_t stream) {
  if (p.M_pad % 128 != 0 || p.K % 128 != 0) return cudaErrorInvalidValue;
  if (fmt == SVDQ_INT4_G64) return launch_fmt<SVDQ_INT4_G64>(p, rp, stream);
  return launch_fmt<SVDQ_NVFP4_G16>(p, rp, stream);
}

}  // namespace svdq
