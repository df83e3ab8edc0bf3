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
// Persistent kernel, one CTA per SM, 128 x 256 output tiles taken round-robin.
// Warp roles (11 warps):
//   warp 0  producer: for each tile, a bulk copy of the bias slice, then the
//           k-tiles (A and B codes by TMA, their scale-factor atoms by bulk
//           copy) followed by the branch k-tiles (a 32-column slice of T'
//           and of L2^T), through a 4-stage shared-memory ring;
//   warp 10 scale factors: copies each stage's scale-factor atoms into that
//           stage's TMEM slot with tcgen05.cp and commits them to the stage's
//           sf_ready barrier. Copies issued from the MMA thread serialise
//           with its MMAs (about 47 cycles per copy, 12 per k-tile, against
//           512 cycles of MMAs); from a thread of their own they overlap;
//   warp 1  TMEM owner and MMA issuer (one thread): per k-tile, once the
//           stage's scale factors are in TMEM, 4 block-scaled MMAs; per
//           branch k-tile 2 kind::f16 MMAs; commits release the stage / mark
//           the tile;
//   warps 2-9 epilogue: each copies its 32 rows x 128 columns of the
//           accumulator to registers and releases TMEM at once, so the next
//           tile's MMAs overlap the scaling, bias and bf16 stores.
// Tiles are ordered with the N index fastest so the CTAs in flight share the
// weight panel in L2.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBKBytes = 128;  // 256 E2M1 values per row per k-tile
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kCpWarp = 2 + kEpiWarps;  // copies scale factors into TMEM
constexpr int kThreads = (3 + kEpiWarps) * 32;

struct SmemNv {
  static constexpr int kA = kBM * kBKBytes;   // 16 KB
  static constexpr int kB = kBN * kBKBytes;   // 32 KB
  static constexpr int kSfa = 4 * 512;        // 4 k-blocks of 64
  static constexpr int kSfb = (kBN / 128) * 4 * 512;
  static constexpr int kStage = kA + kB + kSfa + kSfb;
  static constexpr int kBiasOff = kStages * kStage;
  static constexpr int kBias = kBN * 2;       // bf16 bias slice of a tile
  static constexpr int kBarOff = kBiasOff + 2 * kBias;
  static constexpr int kTotal = kBarOff + 256 + 1024;
};
static_assert(SmemNv::kTotal <= 232448, "shared memory budget");
static_assert(kBN % kWeightBoxRows == 0 && kBM % kActBoxRows == 0, "operand tiles are whole boxes");

// TMEM columns: accumulator [0, 256), then one scale-factor slot per
// shared-memory stage (A: 16 columns, B: 32), so copying the next k-tile's
// scale factors never waits for the MMAs still reading the previous ones.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfSlotCols = 16 + 2 * 16;
constexpr uint32_t kSfaCol = kBN;
constexpr uint32_t kSfbCol = kBN + 16;
static_assert(kBN + kStages * kSfSlotCols <= kTmemCols, "TMEM budget");

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const GemmParams p, const __grid_constant__ GemmMaps maps) {
  using L = SmemNv;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* bias_full = acc_empty + 1;   // [2]
  uint64_t* bias_empty = bias_full + 2;  // [2]
  uint64_t* drain = bias_empty + 2;
  uint64_t* sf_ready = drain + 1;        // [kStages] scale factors of the stage are in TMEM
  uint64_t* cp_done = sf_ready + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cp_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.N + kBN - 1) / kBN;
  const int n_tiles = (p.M_pad / kBM) * n_blocks;
  const int kb_total = p.K / 64;
  const int n_main = (p.K + 255) / 256;
  const int n_lr = p.RP / 32;
  const int n_items = n_main + n_lr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bias_full[b], 1);
      mbar_init(&bias_empty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < kStages; ++s) mbar_init(&sf_ready[s], 1);
    mbar_init(cp_done, 1);
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
    if (lane == 0) {
      prefetch_tensormap(&maps.a);
      prefetch_tensormap(&maps.b);
      if (n_lr > 0) {  // no branch (rank 0): its maps are never read
        prefetch_tensormap(&maps.t);
        prefetch_tensormap(&maps.l2);
      }
      bool ok = true;
      int it = 0;          // k-tiles issued over all tiles of this CTA
      int ti = 0;          // tiles of this CTA
      int last_bias = -1;  // last tile whose bias copy was issued
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++ti) {
        const int mb = tile / n_blocks, nb = tile % n_blocks;
        const int m0 = mb * kBM, n0 = nb * kBN;
        const int bs = ti & 1;
        ok = mbar_wait(&bias_empty[bs], ((ti >> 1) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        mbar_arrive_expect_tx(&bias_full[bs], L::kBias);
        bulk_load(smem + L::kBiasOff + bs * L::kBias, p.bias + n0, L::kBias, &bias_full[bs]);
        last_bias = ti;
        for (int k = 0; k < n_items && ok; ++k, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          uint8_t* st = smem + s * L::kStage;
          if (k < n_main) {
            const int kb0 = k * 4;
            const int nkb = min(4, kb_total - kb0);
            mbar_arrive_expect_tx(&full[s], L::kA + L::kB + nkb * 512 * (1 + kBN / 128));
#pragma unroll
            for (int h = 0; h < kBM / kActBoxRows; ++h)
              tma_load_2d(st + h * kActBoxRows * kBKBytes, &maps.a, &full[s], k * kBKBytes, m0 + h * kActBoxRows);
#pragma unroll
            for (int h = 0; h < kBN / kWeightBoxRows; ++h)
              tma_load_2d(st + L::kA + h * kWeightBoxRows * kBKBytes, &maps.b, &full[s], k * kBKBytes, n0 + h * kWeightBoxRows);
            const uint8_t* sa = reinterpret_cast<const uint8_t*>(p.sa) + (static_cast<size_t>(mb) * kb_total + kb0) * 512;
            bulk_load(st + L::kA + L::kB, sa, nkb * 512, &full[s]);
#pragma unroll
            for (int h = 0; h < kBN / 128; ++h) {
              const uint8_t* sb = reinterpret_cast<const uint8_t*>(p.sb) +
                                  (static_cast<size_t>(nb * (kBN / 128) + h) * kb_total + kb0) * 512;
              bulk_load(st + L::kA + L::kB + L::kSfa + h * 2048, sb, nkb * 512, &full[s]);
            }
          } else {
            const int c = k - n_main;  // 32-column slice of the branch
            mbar_arrive_expect_tx(&full[s], kBM * 64 + kBN * 64);
            tma_load_2d(st, &maps.t, &full[s], c * 32, m0);
#pragma unroll
            for (int h = 0; h < kBN / kWeightBoxRows; ++h)
              tma_load_2d(st + L::kA + h * kWeightBoxRows * 64, &maps.l2, &full[s], c * 32,
                          n0 + h * kWeightBoxRows);
          }
        }
      }
      if (!ok) {
        // gave up: let the copies already in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int j = max(0, it - kStages); j < it; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1, &no_abort, nullptr);
        for (int t2 = last_bias - 1; t2 <= last_bias; ++t2)
          if (t2 >= 0) mbar_wait(&bias_full[t2 & 1], (t2 >> 1) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_main = idesc_block_scaled(kBM, kBN);
    const uint32_t idesc_lr = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kBM, kBN);
    bool ok = true;
    int it = 0, ti = 0;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++ti) {
      // the epilogue has copied the previous tile's accumulator out of TMEM
      ok = mbar_wait(acc_empty, (ti & 1) ^ 1, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      for (int k = 0; k < n_items && ok; ++k, ++it) {
        const int s = it % kStages;
        ok = mbar_wait(&sf_ready[s], (it / kStages) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {  // one fixed thread issues every tcgen05 op, so its commits track them all
          uint8_t* st = smem + s * L::kStage;
          const uint32_t a_base = smem_u32(st);
          const uint32_t b_base = smem_u32(st + L::kA);
          if (k < n_main) {
            const int nkb = min(4, kb_total - k * 4);
            const uint32_t t_sfa = tmem + kSfaCol + s * kSfSlotCols;
            const uint32_t t_sfb = tmem + kSfbCol + s * kSfSlotCols;
            for (int j = 0; j < nkb; ++j) {
              const uint64_t ad = smem_desc(a_base + 32 * j, 16, 1024, kSw128);
              const uint64_t bd = smem_desc(b_base + 32 * j, 16, 1024, kSw128);
              mma_nvf4(tmem, ad, bd, idesc_main, t_sfa + 4 * j, t_sfb + (kBN / 32) * j, (k > 0 || j > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint64_t ad = smem_desc(a_base + 32 * j, 16, 512, kSw64);
              const uint64_t bd = smem_desc(b_base + 32 * j, 16, 512, kSw64);
              mma_f16(tmem, ad, bd, idesc_lr, 1u);
            }
          }
          tc_commit(&empty[s]);
          if (k == n_items - 1) tc_commit(acc_full);
        }
        __syncwarp();
      }
    }
  } else if (warp == kCpWarp) {
    // ------------------------------------------------------------ scale factors to TMEM
    // One stage ahead of the MMA thread at most (it waits for each stage's
    // copies): the copies and the MMAs come from different threads.
    if (lane == 0) {
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        for (int k = 0; k < n_items && ok; ++k, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&full[s], (it / kStages) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          if (k < n_main) {
            uint8_t* st = smem + s * L::kStage;
            const int nkb = min(4, kb_total - k * 4);
            const uint32_t t_sfa = tmem + kSfaCol + s * kSfSlotCols;
            const uint32_t t_sfb = tmem + kSfbCol + s * kSfSlotCols;
            const uint32_t sfa_base = smem_u32(st + L::kA + L::kB);
            const uint32_t sfb_base = sfa_base + L::kSfa;
            for (int j = 0; j < nkb; ++j) {
              tmem_cp_32x128b_x4(t_sfa + 4 * j, smem_desc(sfa_base + 512 * j, 16, 128, kSwNone));
#pragma unroll
              for (int h = 0; h < kBN / 128; ++h)
                tmem_cp_32x128b_x4(t_sfb + (kBN / 32) * j + 4 * h,
                                   smem_desc(sfb_base + h * 2048 + 512 * j, 16, 128, kSwNone));
            }
          }
          tc_commit(&sf_ready[s]);
        }
      }
      tc_commit(cp_done);  // arrives once every copy issued above has finished
      volatile int no_abort = 0;
      mbar_wait(cp_done, 0, &no_abort, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                  // 0..7
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int col0 = (ew >> 2) * (kBN / 2);   // this warp's half of the tile's columns
    bool ok = true;
    int ti = 0;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++ti) {
      const int mb = tile / n_blocks, nb = tile % n_blocks;
      const int row = mb * kBM + 32 * q + lane;
      const int nbase = nb * kBN + col0;
      ok = mbar_wait(acc_full, ti & 1, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      uint32_t r[kBN / 2];
      const uint32_t ta = tmem + (static_cast<uint32_t>(32 * q) << 16) + col0;
#pragma unroll
      for (int c = 0; c < kBN / 64; ++c) tmem_ld32(ta + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);  // TMEM free for the next tile's MMAs
      const int bs = ti & 1;
      ok = mbar_wait(&bias_full[bs], (ti >> 1) & 1, abort_flag, p.status);
      if (!ok) break;
      const uint32_t* bias = reinterpret_cast<const uint32_t*>(smem + L::kBiasOff + bs * L::kBias) + col0 / 2;
      if (row < p.M) {
#pragma unroll
        for (int v = 0; v < kBN / 16; ++v) {
          const int n = nbase + 8 * v;
          if (n < p.N) {
            const uint4 bw = *reinterpret_cast<const uint4*>(bias + 4 * v);
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&bias_empty[bs]);
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

}  // namespace


cudaError_t launch_gemm_nvfp4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemNv::kTotal);
  });
  if (e != cudaSuccess) return e;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int tiles = (p.M_pad / kBM) * ((p.N + kBN - 1) / kBN);
  const int grid = tiles < sms ? tiles : sms;
  gemm_nvfp4_kernel<<<grid, kThreads, SmemNv::kTotal, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace svdq
