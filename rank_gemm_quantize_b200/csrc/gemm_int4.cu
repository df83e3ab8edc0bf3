// K3: INT4 (group 64) W4A4 GEMM with the low-rank branch and the bias fused in.
//
// Computes, for one SVDQuant linear layer ("SVDQuant: Absorbing Outliers by
// Low-Rank Components for 4-Bit Diffusion Models", abstract; msModelSlim
// SVDQuant entry, section 2.3, the dual-path output equation):
//   Y[m,n] = sum_g sx[m,g] sw[n,g] sum_{k in g} qx[m,k] qw[n,k]  +  (T L2)[m,n]  + b[n]
// B200 has no 4-bit integer tensor-core path and no block-scaled MMA with
// arbitrary float32 group scales, so each 64-wide group is contracted exactly
// on its own and rescaled on the CUDA cores:
//  * the integer codes (-8..7) are held as E4M3 bytes, which represent them
//    exactly, and contracted with tcgen05 kind::f8f6f4 (E4M3 x E4M3, fp32
//    accumulation in TMEM; every partial sum is an integer below 2^13, hence
//    exact). Compared with kind::i8 this runs at the same tensor rate and
//    leaves an fp32 result, so the per-group rescale needs no int->float
//    conversion;
//  * four TMEM accumulators rotate between groups: the tensor core runs up to
//    three groups ahead while the epilogue warps drain group g and accumulate
//    sx * sw * D into registers;
//  * after the last group the branch product T L2 (kind::f16, bf16 in, fp32
//    out) goes through the same ping-pong buffer, then bias and one bf16 store.
//
// CTA = 18 warps: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps
// 2-17 drain/epilogue, each owning one 32-lane TMEM quarter (32 output rows)
// and 32 of the tile's columns, with its fp32 accumulators in registers. Four
// drain warps per SM sub-partition hide each other's TMEM-load latency; the
// drain of a group costs about as many issue slots as its MMA takes cycles.
// The rescale uses the packed fp32x2 multiply / fma of sm_100 (two outputs per
// instruction); the per-group scales of both operands arrive in a small shared
// memory ring filled by the producer's bulk copies.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // bytes (= codes) per row per k-tile: two groups of 64
constexpr int kDrainWarps = 16;
constexpr int kFirstDrainWarp = 2;
constexpr int kThreads = (kFirstDrainWarp + kDrainWarps) * 32;
// Ring of per-group scale vectors (weights then activations). It is deep so
// that the producer's lookahead is bounded by the data ring, not by the
// slowest drain warp.
constexpr int kSwSlots = 32;
constexpr int kDBufs = 4;    // TMEM accumulators the groups rotate through

template <int BN, int STAGES>
struct SmemI4 {
  static constexpr int kA = kBM * kBK;  // 16 KB
  static constexpr int kB = BN * kBK;
  static constexpr int kStage = kA + kB;
  static constexpr int kSlot = (BN + kBM) * 4;  // sw[BN] then sx[BM]
  static constexpr int kSwOff = STAGES * kStage;
  static constexpr int kBarOff = kSwOff + kSwSlots * kSlot;
  static constexpr int kBarBytes = (2 * STAGES + 2 * kSwSlots + 2 * kDBufs + 1) * 8 + 16;
  static constexpr int kTotal = kBarOff + ((kBarBytes + 127) / 128) * 128 + 1024;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_int4_kernel(const GemmParams p, const __grid_constant__ GemmMaps maps) {
  using L = SmemI4<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sw_ring = reinterpret_cast<float*>(smem + L::kSwOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* sw_full = empty + STAGES;
  uint64_t* sw_empty = sw_full + kSwSlots;
  uint64_t* d_full = sw_empty + kSwSlots;   // [kDBufs]
  uint64_t* d_empty = d_full + kDBufs;      // [kDBufs]
  uint64_t* drain = d_empty + kDBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.N + BN - 1) / BN;
  const int mb = blockIdx.x / n_blocks;
  const int nb = blockIdx.x % n_blocks;
  const int m0 = mb * kBM, n0 = nb * BN;
  const int n_groups = p.K / 64;
  const int n_main = (p.K + kBK - 1) / kBK;
  const int n_lr = p.RP / 32;
  const int n_items = n_main + n_lr;
  constexpr uint32_t kTmemCols = 512;
  static_assert(BN % 64 == 0 && kDBufs * BN <= 512, "tile width");

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kSwSlots; ++s) {
      mbar_init(&sw_full[s], 1);
      mbar_init(&sw_empty[s], kDrainWarps);
    }
    for (int b = 0; b < kDBufs; ++b) {
      mbar_init(&d_full[b], 1);
      mbar_init(&d_empty[b], kDrainWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      prefetch_tensormap(&maps.a);
      prefetch_tensormap(&maps.b);
      prefetch_tensormap(&maps.t);
      prefetch_tensormap(&maps.l2);
      int it = 0;
      bool ok = true;
      for (; it < n_items && ok; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (it < n_main) {
          // per-group weight scales of this k-tile (released by the epilogue)
          for (int gg = 0; gg < 2 && ok; ++gg) {
            const int g = 2 * it + gg;
            if (g >= n_groups) break;
            const int ws = g % kSwSlots;
            ok = mbar_wait(&sw_empty[ws], ((g / kSwSlots) & 1) ^ 1, abort_flag, p.status);
            if (!ok) break;
            float* slot = sw_ring + ws * (BN + kBM);
            mbar_arrive_expect_tx(&sw_full[ws], (BN + kBM) * 4);
            bulk_load(slot, reinterpret_cast<const float*>(p.sb) + static_cast<size_t>(g) * p.N_pad + n0, BN * 4,
                      &sw_full[ws]);
            bulk_load(slot + BN, reinterpret_cast<const float*>(p.sa) + static_cast<size_t>(g) * p.M_pad + m0,
                      kBM * 4, &sw_full[ws]);
          }
          if (!ok) break;
        }
        ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, p.status);
        if (!ok) break;
        uint8_t* st = smem + s * L::kStage;
        if (it < n_main) {
          mbar_arrive_expect_tx(&full[s], L::kA + L::kB);
          tma_load_2d(st, &maps.a, &full[s], it * kBK, m0);
          tma_load_2d(st + L::kA, &maps.b, &full[s], it * kBK, n0);
        } else {
          const int c = it - n_main;
          mbar_arrive_expect_tx(&full[s], kBM * 64 + BN * 64);
          tma_load_2d(st, &maps.t, &full[s], c * 32, m0);
          tma_load_2d(st + L::kA, &maps.l2, &full[s], c * 32, n0);
        }
      }
      if (!ok) {
        volatile int no_abort = 0;
        for (int j = max(0, it - STAGES); j < it; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1, &no_abort, nullptr);
        for (int g = max(0, 2 * it - kSwSlots); g < min(n_groups, 2 * it + 2); ++g)
          mbar_wait(&sw_full[g % kSwSlots], (g / kSwSlots) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_q = idesc_dense(kFmtF32, kFmtE4M3, kFmtE4M3, kBM, BN);
    const uint32_t idesc_lr = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kBM, BN);
    bool ok = true;
    for (int it = 0; it < n_items && ok; ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      // the accumulator this k-tile writes: groups 2it, 2it+1, or the branch "group" n_groups
      const bool main_tile = it < n_main;
      if (!main_tile && it == n_main) {
        const int g = n_groups;
        ok = mbar_wait(&d_empty[g % kDBufs], ((g / kDBufs) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
      }
      ok = mbar_wait(&full[s], ph, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * L::kStage);
      const uint32_t b_base = a_base + L::kA;
      if (main_tile) {
        for (int gg = 0; gg < 2; ++gg) {
          const int g = 2 * it + gg;
          if (g >= n_groups) break;
          ok = mbar_wait(&d_empty[g % kDBufs], ((g / kDBufs) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t d = tmem + (g % kDBufs) * BN;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint64_t ad = smem_desc(a_base + 64 * gg + 32 * j, 16, 1024, kSw128);
              const uint64_t bd = smem_desc(b_base + 64 * gg + 32 * j, 16, 1024, kSw128);
              mma_f8f6f4(d, ad, bd, idesc_q, j);
            }
            tc_commit(&d_full[g % kDBufs]);
          }
          __syncwarp();
        }
        if (!ok) break;
      } else {
        if (lane == 0) {
          const int g = n_groups;
          const uint32_t d = tmem + (g % kDBufs) * BN;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint64_t ad = smem_desc(a_base + 32 * j, 16, 512, kSw64);
            const uint64_t bd = smem_desc(b_base + 32 * j, 16, 512, kSw64);
            mma_f16(d, ad, bd, idesc_lr, (it > n_main || j > 0) ? 1u : 0u);
          }
          if (it == n_items - 1) tc_commit(&d_full[g % kDBufs]);
        }
        __syncwarp();
      }
      if (lane == 0) tc_commit(&empty[s]);
      __syncwarp();
    }
  } else if (warp >= kFirstDrainWarp) {
    // ------------------------------------------------------------ drain / epilogue
    const int dw = warp - kFirstDrainWarp;   // drain warp 0..15
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    constexpr int kCols = BN / (kDrainWarps / 4);
    const int col0 = (dw >> 2) * kCols;      // this warp's slice of the tile's columns
    const int row = m0 + 32 * q + lane;
    float2 acc[kCols / 2];
#pragma unroll
    for (int j = 0; j < kCols / 2; ++j) acc[j] = make_float2(0.f, 0.f);
    bool ok = true;
    for (int g = 0; g <= n_groups && ok; ++g) {
      const bool branch = (g == n_groups);
      const int ws = g % kSwSlots;
      if (!branch) {
        ok = mbar_wait(&sw_full[ws], (g / kSwSlots) & 1, abort_flag, p.status);
        if (!ok) break;
      }
      ok = mbar_wait(&d_full[g % kDBufs], (g / kDBufs) & 1, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tmem + (g % kDBufs) * BN + col0 + (static_cast<uint32_t>(32 * q) << 16);
      const float* slot = sw_ring + ws * (BN + kBM);
      const float sx = branch ? 1.f : slot[BN + 32 * q + lane];
      const float2 sx2 = make_float2(sx, sx);
      const float4* sw4 = reinterpret_cast<const float4*>(slot + col0);
#pragma unroll
      for (int c = 0; c < kCols / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(d + 32 * c, r);
        tmem_ld_wait();
        if (branch) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            acc[16 * c + j] = __fadd2_rn(acc[16 * c + j], make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])));
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 w = sw4[8 * c + j];
            const float2 w01 = __fmul2_rn(sx2, make_float2(w.x, w.y));
            const float2 w23 = __fmul2_rn(sx2, make_float2(w.z, w.w));
            acc[16 * c + 2 * j] = __ffma2_rn(w01, make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])),
                                             acc[16 * c + 2 * j]);
            acc[16 * c + 2 * j + 1] = __ffma2_rn(
                w23, make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])), acc[16 * c + 2 * j + 1]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&d_empty[g % kDBufs]);
        if (!branch) mbar_arrive(&sw_empty[ws]);
      }
    }
    if (ok && row < p.M) {
#pragma unroll
      for (int v = 0; v < kCols / 8; ++v) {
        const int n = n0 + col0 + 8 * v;
        if (n < p.N) {
          const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
          const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a = acc[4 * v + e];
            const float y0 = a.x + __uint_as_float(bb[e] << 16);
            const float y1 = a.y + __uint_as_float(bb[e] & 0xFFFF0000u);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            o[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(row) * p.N + n) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (lane == 0) tc_commit(drain);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort, nullptr);
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int BN, int STAGES>
cudaError_t launch_bn(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  using L = SmemI4<BN, STAGES>;
  auto kern = gemm_int4_kernel<BN, STAGES>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = (p.M_pad / kBM) * ((p.N + BN - 1) / BN);
  kern<<<grid, kThreads, L::kTotal, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace

int gemm_int4_bn() { return 128; }

cudaError_t launch_gemm_int4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  return launch_bn<128, 4>(p, maps, stream);
}

}  // namespace svdq
