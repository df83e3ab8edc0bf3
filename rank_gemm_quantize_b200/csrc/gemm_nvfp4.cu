// K2: NVFP4 W4A4 GEMM with the low-rank branch and the bias fused in.
//
// Computes, for one SVDQuant linear layer ("SVDQuant: Absorbing Outliers by
// Low-Rank Components for 4-Bit Diffusion Models", abstract; msModelSlim
// SVDQuant entry, section 2.3, the dual-path output equation):
//   Y = g_x g_w * ( sum_k Q(x_hat) Q(R)  +  T' L2 )  + b
// where the 4-bit product runs on tcgen05 kind::mxf4nvf4 block-scaled MMAs
// (E2M1 x E2M1, one UE4M3 scale per 16 elements on each side, fp32
// accumulation in TMEM) and T' = x_hat L1 / (g_x g_w) is the bf16 branch
// input written by the activation kernel. The branch product T' L2 is
// accumulated into the same TMEM accumulator with kind::f16 MMAs, so the
// low-rank term never makes a separate pass over Y; the epilogue applies the
// tensor scales and the bias and stores bf16 once.
//
// CTA = 6 warps: warp 0 issues TMA / bulk copies into a STAGES-deep shared
// memory ring, warp 1 owns TMEM and issues the MMAs (one elected thread),
// warps 2-5 read the accumulator back (one 32-lane TMEM quarter each) and
// write Y. The ring carries ceil(K/256) main k-tiles followed by RP/32
// low-rank k-tiles (a 32-column slice of T' and of L2^T each).
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 E2M1 values per row per k-tile
constexpr int kThreads = 192;

template <int BN, int STAGES>
struct SmemNv {
  static constexpr int kA = kBM * kBKBytes;         // 16 KB
  static constexpr int kB = BN * kBKBytes;
  static constexpr int kSfa = 4 * 512;              // 4 k-blocks of 64
  static constexpr int kSfb = (BN / 128) * 4 * 512;
  static constexpr int kStage = kA + kB + kSfa + kSfb;
  static constexpr int kBarOff = STAGES * kStage;
  static constexpr int kTotal = kBarOff + 256 + 1024;  // barriers + alignment slack
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const GemmParams p, const __grid_constant__ GemmMaps maps) {
  using L = SmemNv<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.N + BN - 1) / BN;
  const int mb = blockIdx.x / n_blocks;
  const int nb = blockIdx.x % n_blocks;
  const int m0 = mb * kBM, n0 = nb * BN;
  const int kb_total = p.K / 64;
  const int n_main = (p.K + 255) / 256;
  const int n_lr = p.RP / 32;
  const int n_items = n_main + n_lr;
  constexpr uint32_t kTmemCols = (BN + 16 + BN / 8) <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
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
  const uint32_t t_acc = tmem;
  const uint32_t t_sfa = tmem + BN;
  const uint32_t t_sfb = tmem + BN + 16;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      prefetch_tensormap(&maps.a);
      prefetch_tensormap(&maps.b);
      prefetch_tensormap(&maps.t);
      prefetch_tensormap(&maps.l2);
      int it = 0;
      for (; it < n_items; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.status)) break;
        uint8_t* st = smem + s * L::kStage;
        if (it < n_main) {
          const int kb0 = it * 4;
          const int nkb = min(4, kb_total - kb0);
          const uint32_t bytes = L::kA + L::kB + nkb * 512 * (1 + BN / 128);
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(st, &maps.a, &full[s], it * kBKBytes, m0);
          tma_load_2d(st + L::kA, &maps.b, &full[s], it * kBKBytes, n0);
          const uint8_t* sa = reinterpret_cast<const uint8_t*>(p.sa) + (static_cast<size_t>(mb) * kb_total + kb0) * 512;
          bulk_load(st + L::kA + L::kB, sa, nkb * 512, &full[s]);
#pragma unroll
          for (int h = 0; h < BN / 128; ++h) {
            const uint8_t* sb = reinterpret_cast<const uint8_t*>(p.sb) +
                                (static_cast<size_t>(nb * (BN / 128) + h) * kb_total + kb0) * 512;
            bulk_load(st + L::kA + L::kB + L::kSfa + h * 2048, sb, nkb * 512, &full[s]);
          }
        } else {
          const int c = it - n_main;  // 32-column slice of the branch
          mbar_arrive_expect_tx(&full[s], kBM * 64 + BN * 64);
          tma_load_2d(st, &maps.t, &full[s], c * 32, m0);
          tma_load_2d(st + L::kA, &maps.l2, &full[s], c * 32, n0);
        }
      }
      if (it < n_items) {
        // gave up: let the copies already in flight land before the CTA exits
        for (int j = max(0, it - STAGES); j < it; ++j) {
          volatile int no_abort = 0;
          mbar_wait(&full[j % STAGES], (j / STAGES) & 1, &no_abort, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_main = idesc_block_scaled(kBM, BN);
    const uint32_t idesc_lr = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kBM, BN);
    bool ok = true;
    for (int it = 0; it < n_items && ok; ++it) {
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      ok = mbar_wait(&full[s], ph, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {  // one fixed thread issues every tcgen05 op, so its commits track them all
        uint8_t* st = smem + s * L::kStage;
        const uint32_t a_base = smem_u32(st);
        const uint32_t b_base = smem_u32(st + L::kA);
        if (it < n_main) {
          const int nkb = min(4, kb_total - it * 4);
          const uint32_t sfa_base = smem_u32(st + L::kA + L::kB);
          const uint32_t sfb_base = sfa_base + L::kSfa;
          for (int j = 0; j < nkb; ++j) {
            tmem_cp_32x128b_x4(t_sfa + 4 * j, smem_desc(sfa_base + 512 * j, 16, 128, kSwNone));
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              tmem_cp_32x128b_x4(t_sfb + (BN / 32) * j + 4 * h,
                                 smem_desc(sfb_base + h * 2048 + 512 * j, 16, 128, kSwNone));
          }
          for (int j = 0; j < nkb; ++j) {
            const uint64_t ad = smem_desc(a_base + 32 * j, 16, 1024, kSw128);
            const uint64_t bd = smem_desc(b_base + 32 * j, 16, 1024, kSw128);
            mma_nvf4(t_acc, ad, bd, idesc_main, t_sfa + 4 * j, t_sfb + (BN / 32) * j, (it > 0 || j > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint64_t ad = smem_desc(a_base + 32 * j, 16, 512, kSw64);
            const uint64_t bd = smem_desc(b_base + 32 * j, 16, 512, kSw64);
            mma_f16(t_acc, ad, bd, idesc_lr, 1u);
          }
        }
        tc_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (ok && lane == 0) tc_commit(acc_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = m0 + 32 * q + lane;
    if (mbar_wait(acc_full, 0, abort_flag, p.status)) {
      tc_fence_after();
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_acc + (static_cast<uint32_t>(32 * q) << 16) + 32 * c, r);
        tmem_ld_wait();
        const int nc = n0 + 32 * c;
        if (row < p.M) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int n = nc + 8 * v;
            if (n < p.N) {
              const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
              const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float b0 = __uint_as_float(bb[e] << 16);
                const float b1 = __uint_as_float(bb[e] & 0xFFFF0000u);
                const float y0 = fmaf(__uint_as_float(r[8 * v + 2 * e]), p.out_scale, b0);
                const float y1 = fmaf(__uint_as_float(r[8 * v + 2 * e + 1]), p.out_scale, b1);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
                o[e] = *reinterpret_cast<uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(row) * p.N + n) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (lane == 0) tc_commit(drain);  // arrives once every tcgen05 op issued by lane 0 has finished
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort, nullptr);
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int BN, int STAGES>
cudaError_t launch_bn(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  using L = SmemNv<BN, STAGES>;
  auto kern = gemm_nvfp4_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
  if (e != cudaSuccess) return e;
  const int grid = (p.M_pad / kBM) * ((p.N + BN - 1) / BN);
  kern<<<grid, kThreads, L::kTotal, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace

int gemm_nvfp4_bn() { return 128; }

cudaError_t launch_gemm_nvfp4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  return launch_bn<128, 4>(p, maps, stream);
}

}  // namespace svdq
