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
// Work split: a thread-block cluster of S CTAs owns 64 rows; CTA r of the
// cluster walks its 1/S share of K in 64-column chunks (S is chosen so the
// grid covers the SMs once and every cluster is resident). Per chunk:
//   * warp 17 (one thread) streams the X tile [64 x 64], the L1^T slice
//     [RP x 64] and the inv_s slice into a shared-memory ring with TMA / bulk
//     copies (128-byte swizzle);
//   * warps 0-15 (4 rows each) smooth, quantize, store codes and scales, and
//     write x_hat as a bf16 high part and a bf16 remainder straight into a
//     tcgen05 K-major operand buffer (128 rows: the MMA's M; rows 64-127 stay
//     zero and their results are ignored);
//   * one thread of warp 16 then issues tcgen05 kind::f16 MMAs
//     (M = 128, N = RP, bf16 x bf16 -> fp32) of hi and lo against L1 into a
//     TMEM accumulator, so T's only sizable error is its final bf16 store.
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

constexpr int kRows = 64;      // rows per cluster
constexpr int kMmaM = 128;     // tcgen05 M; operand rows >= kRows are zero
constexpr int kQWarps = 16;    // quantizing warps, 4 rows each
constexpr int kMmaWarp = kQWarps;      // TMEM owner + MMA issuer
constexpr int kProdWarp = kQWarps + 1; // TMA producer
constexpr int kThreads = (kQWarps + 2) * 32;
constexpr int kPair = 1;               // chunks each quantizing warp processes per iteration
constexpr int kChunk = 64;     // columns per chunk (one 128-byte swizzle atom of bf16)
constexpr int kRedCols = 64;   // columns per cluster-reduction pass

template <int RP>
struct K1Shape {
  static constexpr int kStages = RP <= 64 ? 4 : (RP <= 224 ? 3 : 2);
  // x_hat operand buffers: phase A runs up to this many chunks ahead of the MMA
  static constexpr int kABufs = RP <= 128 ? 4 : 3;
  static constexpr int kX = kRows * 128;             // X tile of a chunk (bf16, 64 cols)
  static constexpr int kL = RP * 128;                // L1^T slice of a chunk
  static constexpr int kS = 1024;                    // inv_s slice of a chunk (256 B used, 1 KB keeps alignment)
  static constexpr int kStage = kX + kL + kS;
  static constexpr int kAHalf = kMmaM * 128;         // one operand (hi or lo) of a chunk
  static constexpr int kA = 2 * kAHalf;              // hi + lo MMA operand of a chunk
  static constexpr int kAOff = kStages * kStage;
  static constexpr int kRedOff = kAOff + kABufs * kA;
  static constexpr int kRedW = RP < kRedCols ? RP : kRedCols;
  static constexpr int kRed = kRows * kRedW * 4;
  static constexpr int kBarOff = kRedOff + kRed;
  static constexpr int kTotal = kBarOff + 256 + 1024;
  static_assert(kTotal <= 232448, "shared memory budget");
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

// Quantize NP independent sets of 8 consecutive smoothed values (each one
// lane's share of a group in a different row or chunk), stage by stage so the
// NP dependency chains interleave; then store the codes and, from one lane per
// group, the group scales.
template <int FMT, int NP>
__device__ __forceinline__ void quantize_passes(const float (&v)[NP][8], const ActQuantParams& p, const int (&row)[NP],
                                                const int (&k)[NP], int cs) {
  float amax[NP];
#pragma unroll
  for (int u = 0; u < NP; ++u) {
    const float m01 = fmaxf(fabsf(v[u][0]), fabsf(v[u][1])), m23 = fmaxf(fabsf(v[u][2]), fabsf(v[u][3]));
    const float m45 = fmaxf(fabsf(v[u][4]), fabsf(v[u][5])), m67 = fmaxf(fabsf(v[u][6]), fabsf(v[u][7]));
    amax[u] = fmaxf(fmaxf(m01, m23), fmaxf(m45, m67));
  }
  if (FMT == SVDQ_INT4_G64) {
    // group of 64 = the 8 lanes sharing (lane >> 3)
#pragma unroll
    for (int o = 1; o <= 4; o <<= 1)
#pragma unroll
      for (int u = 0; u < NP; ++u) amax[u] = fmaxf(amax[u], __shfl_xor_sync(0xffffffffu, amax[u], o));
    float scale[NP], inv[NP];
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      const float safe = amax[u] > 0.f ? amax[u] : 1.f;
      scale[u] = amax[u] > 0.f ? __fdiv_rn(safe, 7.0f) : 0.f;
      inv[u] = __fdiv_rn(7.0f, safe);
    }
    uint32_t lo[NP], hi[NP];
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      // |v| <= amax and inv <= (7 / amax)(1 + 2^-24), so |v * inv| rounds to at
      // most 7: rint already lands in [-7, 7] and the [-8, 7] clamp never acts.
      // An all-zero group gives v = 0 and codes 0 with the placeholder inv.
      // The rounding must see the float-rounded product: an add-based
      // round-to-integer (adding and subtracting 1.5 * 2^23) gets fused with
      // the multiply into one FMA by the code generator, which rounds the exact
      // product instead and flips products that land exactly on a half.
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 pr = __fmul2_rn(make_float2(v[u][j], v[u][j + 1]), make_float2(inv[u], inv[u]));
        q[j] = rintf(pr.x);
        q[j + 1] = rintf(pr.y);
      }
      lo[u] = cvt_e4m3x2(q[0], q[1]) | (cvt_e4m3x2(q[2], q[3]) << 16);
      hi[u] = cvt_e4m3x2(q[4], q[5]) | (cvt_e4m3x2(q[6], q[7]) << 16);
    }
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      *reinterpret_cast<uint2*>(p.codes + static_cast<size_t>(row[u]) * p.K + k[u]) = make_uint2(lo[u], hi[u]);
      if (cs == 0) reinterpret_cast<float*>(p.scales)[static_cast<size_t>(k[u] >> 6) * p.M_pad + row[u]] = scale[u];
    }
  } else {
    // group of 16 = this lane and its neighbour (lane ^ 1)
#pragma unroll
    for (int u = 0; u < NP; ++u) amax[u] = fmaxf(amax[u], __shfl_xor_sync(0xffffffffu, amax[u], 1));
    uint32_t sb[NP];
    float eff[NP];
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      sb[u] = cvt_e4m3x2(__fdiv_rn(amax[u], p.denom), 0.f) & 0xFFu;
      eff[u] = __fmul_rn(e4m3_to_float(sb[u]), p.g_x);
    }
    uint32_t codes[NP];
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      const float inv = __frcp_rn(eff[u] != 0.f ? eff[u] : 1.f);
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 pr = __fmul2_rn(make_float2(v[u][j], v[u][j + 1]), make_float2(inv, inv));
        q[j] = pr.x;
        q[j + 1] = pr.y;
      }
      codes[u] = eff[u] != 0.f ? cvt_e2m1x8(q) : 0u;
    }
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      *reinterpret_cast<uint32_t*>(p.codes + static_cast<size_t>(row[u]) * (p.K >> 1) + (k[u] >> 1)) = codes[u];
      if ((cs & 1) == 0) {
        const int sf = k[u] >> 4;  // scale index along the row
        const size_t atom = static_cast<size_t>(row[u] >> 7) * (p.K >> 6) + (sf >> 2);
        const int off = (row[u] & 31) * 16 + ((row[u] >> 5) & 3) * 4 + (sf & 3);
        reinterpret_cast<uint8_t*>(p.scales)[atom * 512 + off] = static_cast<uint8_t>(sb[u]);
      }
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
  uint64_t* aready = empty + S::kStages;                           // [S::kABufs] operand written by warps 0-15
  uint64_t* afree = aready + S::kABufs;                               // [S::kABufs] MMA done reading the operand
  uint64_t* mma_done = afree + S::kABufs;
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
  {
    // operand rows kRows..kMmaM-1 are never written per chunk: clear them once
    uint4* a = reinterpret_cast<uint4*>(smem + S::kAOff);
    const int per_half = (kMmaM - kRows) * 128 / 16;
    for (int i = threadIdx.x; i < 2 * S::kABufs * per_half; i += kThreads) {
      const int half = i / per_half;  // (buffer, hi/lo)
      a[(half * S::kAHalf + kRows * 128) / 16 + (i % per_half)] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
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
      const uint32_t idesc = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kMmaM, RP);
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
    const int cs = lane & 7;   // 16-byte column segment of the chunk
    const int rl = lane >> 3;  // row within a 4-row pass
    const int r0 = warp * (kRows / kQWarps);  // this warp's rows
    bool ok = true;
    for (int j0 = 0; j0 < nlocal && ok; j0 += kPair) {
      const int npair = min(kPair, nlocal - j0);
      for (int u = 0; u < npair && ok; ++u) {
        const int j = j0 + u;
        ok = mbar_wait(&full[j % S::kStages], (j / S::kStages) & 1, abort_flag, p.status);
        if (ok && j >= S::kABufs)
          ok = mbar_wait(&afree[j % S::kABufs], ((j / S::kABufs) & 1) ^ 1, abort_flag, p.status);
      }
      if (!ok) break;
      // The passes of the pair (and of the rows of this warp) are independent:
      // every stage below runs over all of them, so their chains interleave.
      constexpr int kPasses = kRows / kQWarps / 4;  // 4-row passes per chunk
      constexpr int NP = kPair * kPasses;
      float v[NP][8];
      int rows[NP], ks[NP];
      uint8_t* adst[NP];
      int phys[NP];
#pragma unroll
      for (int u = 0; u < kPair; ++u) {
        const int j = j0 + (u < npair ? u : 0);  // a missing second chunk repeats the first (results unused)
        const uint8_t* xt = smem + (j % S::kStages) * S::kStage;
        const float* inv_s = reinterpret_cast<const float*>(xt + S::kX + S::kL) + cs * 8;
        const float4 is0 = *reinterpret_cast<const float4*>(inv_s);
        const float4 is1 = *reinterpret_cast<const float4*>(inv_s + 4);
#pragma unroll
        for (int i = 0; i < kPasses; ++i) {
          const int n = u * kPasses + i;
          const int lrow = r0 + 4 * i + rl;
          phys[n] = lrow * 128 + (cs ^ (lrow & 7)) * 16;
          rows[n] = m0 + lrow;
          ks[n] = (c_begin + j) * kChunk + cs * 8;
          adst[n] = smem + S::kAOff + (j % S::kABufs) * S::kA;
          const uint4 xv = *reinterpret_cast<const uint4*>(xt + phys[n]);
          const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
          const float is[8] = {is0.x, is0.y, is0.z, is0.w, is1.x, is1.y, is1.z, is1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // one IEEE round-to-nearest product per element (packed pair)
            const float2 pr = __fmul2_rn(make_float2(bf16_lo(w[e]), bf16_hi(w[e])), make_float2(is[2 * e], is[2 * e + 1]));
            v[n][2 * e] = pr.x;
            v[n][2 * e + 1] = pr.y;
          }
        }
      }
      if (npair == kPair) {
        quantize_passes<FMT, NP>(v, p, rows, ks, cs);
      } else {
        float v1[kPasses][8];
        int rows1[kPasses], ks1[kPasses];
#pragma unroll
        for (int n = 0; n < kPasses; ++n) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v1[n][e] = v[n][e];
          rows1[n] = rows[n];
          ks1[n] = ks[n];
        }
        quantize_passes<FMT, kPasses>(v1, p, rows1, ks1, cs);
      }
#pragma unroll
      for (int n = 0; n < NP; ++n) {
        if (n < npair * kPasses) {
          uint32_t h[4], l[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            h[e] = pack_bf16x2(v[n][2 * e], v[n][2 * e + 1]);  // high parts, one packed conversion
            // the remainders are exact in float: v - bf16(v) has at most 16 significant bits
            const float2 d = __fadd2_rn(make_float2(v[n][2 * e], v[n][2 * e + 1]),
                                        make_float2(-bf16_lo(h[e]), -bf16_hi(h[e])));
            l[e] = pack_bf16x2(d.x, d.y);
          }
          // same 128-byte swizzle as the TMA tiles: the canonical tcgen05 K-major layout
          *reinterpret_cast<uint4*>(adst[n] + phys[n]) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(adst[n] + S::kAHalf + phys[n]) = make_uint4(l[0], l[1], l[2], l[3]);
        }
      }
      fence_async_smem();  // make the generic-proxy writes visible to the tensor core
      __syncwarp();
      if (lane == 0)
        for (int u = 0; u < npair; ++u) mbar_arrive(&aready[(j0 + u) % S::kABufs]);
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
      if (half * 32 < S::kRedW && q * 32 < kRows) {
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
  if (warp == kMmaWarp) {
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
