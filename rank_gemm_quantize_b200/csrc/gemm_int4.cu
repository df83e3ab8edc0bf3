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
//  * two TMEM accumulators of 128 x 256 alternate between groups: the tensor
//    core contracts group g+1 while the drain warps copy group g out of TMEM
//    and accumulate sx * sw * D into registers;
//  * after the last group the branch product T L2 (kind::f16, bf16 in, fp32
//    out) goes through the same accumulators, then the bias and one bf16
//    store.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles taken round-robin
// with the N index fastest (the CTAs in flight share the weight panel in L2).
// The wide tile halves the shared-memory bytes fetched per MAC compared with
// 128 x 128, which the 8-bit operands need to keep the loads off the critical
// path. Warp roles (18 warps):
//   warp 0      producer: per k-tile (two groups) the A and B codes by TMA
//               into a 4-stage ring, and per group the weight and activation
//               scale vectors by bulk copy into a scale ring; then the
//               branch k-tiles (T and L2^T slices);
//   warp 1      TMEM owner and MMA issuer (one thread): two f8f6f4 MMAs per
//               group into the free accumulator, one commit per group;
//   warps 2-17  drain / epilogue: each owns one 32-lane TMEM quarter (32
//               output rows) and 64 of the tile's columns, with its fp32
//               accumulators in registers (the rescale uses the packed fp32x2
//               multiply / fma of sm_100: two outputs per instruction). A
//               warp releases the TMEM accumulator as soon as its last load
//               of the group has landed, before the arithmetic; at the end of
//               a tile it adds the bias and stores bf16 while the tensor core
//               already runs the next tile.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 128;  // bytes (= codes) per row per k-tile: two groups of 64
constexpr int kStages = 4;
constexpr int kDrainWarps = 16;
constexpr int kFirstDrainWarp = 2;
constexpr int kThreads = (kFirstDrainWarp + kDrainWarps) * 32;
constexpr int kCols = kBN / (kDrainWarps / 4);  // columns per drain warp (64)
// Ring of per-group scale vectors (weights then activations), deep enough that
// the producer's lookahead is bounded by the data ring.
constexpr int kSwSlots = 8;
constexpr int kDBufs = 2;  // TMEM accumulators the groups alternate between
constexpr uint32_t kTmemCols = 512;
static_assert(kDBufs * kBN <= static_cast<int>(kTmemCols), "TMEM budget");
static_assert(kCols % 8 == 0, "drain chunking");

struct SmemI4 {
  static constexpr int kA = kBM * kBK;  // 16 KB
  static constexpr int kB = kBN * kBK;  // 32 KB
  static constexpr int kStage = kA + kB;
  static constexpr int kSlot = (kBN + kBM) * 4;  // sw[BN] then sx[BM]
  static constexpr int kSwOff = kStages * kStage;
  static constexpr int kBarOff = kSwOff + kSwSlots * kSlot;
  static constexpr int kBarBytes = (2 * kStages + 2 * kSwSlots + 2 * kDBufs + 1) * 8 + 16;
  static constexpr int kTotal = kBarOff + ((kBarBytes + 127) / 128) * 128 + 1024;
};
static_assert(SmemI4::kTotal <= 232448, "shared memory budget");
static_assert(kBN % kWeightBoxRows == 0 && kBM % kActBoxRows == 0, "operand tiles are whole boxes");

__global__ void __launch_bounds__(kThreads, 1)
    gemm_int4_kernel(const GemmParams p, const __grid_constant__ GemmMaps maps) {
  using L = SmemI4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sw_ring = reinterpret_cast<float*>(smem + L::kSwOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* sw_full = empty + kStages;
  uint64_t* sw_empty = sw_full + kSwSlots;
  uint64_t* d_full = sw_empty + kSwSlots;  // [kDBufs]
  uint64_t* d_empty = d_full + kDBufs;     // [kDBufs]
  uint64_t* drain = d_empty + kDBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.N + kBN - 1) / kBN;
  const int n_tiles = (p.M_pad / kBM) * n_blocks;
  const int n_groups = p.K / 64;
  const int n_main = p.K / kBK;
  const int n_lr = p.RP / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
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
    if (lane == 0) {
      prefetch_tensormap(&maps.a);
      prefetch_tensormap(&maps.b);
      if (n_lr > 0) {  // no branch (rank 0): its maps are never read
        prefetch_tensormap(&maps.t);
        prefetch_tensormap(&maps.l2);
      }
      bool ok = true;
      int it = 0;  // k-tiles issued by this CTA over all its tiles
      int gs = 0;  // scale vectors issued by this CTA over all its tiles
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / n_blocks) * kBM, n0 = (tile % n_blocks) * kBN;
        for (int k = 0; k < n_main + n_lr && ok; ++k, ++it) {
          if (k < n_main) {
            // the per-group scales of this k-tile (released by the drain warps)
            for (int gg = 0; gg < 2 && ok; ++gg, ++gs) {
              const int g = 2 * k + gg;
              const int ws = gs % kSwSlots;
              ok = mbar_wait(&sw_empty[ws], ((gs / kSwSlots) & 1) ^ 1, abort_flag, p.status);
              if (!ok) break;
              float* slot = sw_ring + ws * (kBN + kBM);
              mbar_arrive_expect_tx(&sw_full[ws], (kBN + kBM) * 4);
              bulk_load(slot, reinterpret_cast<const float*>(p.sb) + static_cast<size_t>(g) * p.N_pad + n0, kBN * 4,
                        &sw_full[ws]);
              bulk_load(slot + kBN, reinterpret_cast<const float*>(p.sa) + static_cast<size_t>(g) * p.M_pad + m0,
                        kBM * 4, &sw_full[ws]);
            }
            if (!ok) break;
          }
          const int s = it % kStages;
          ok = mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          uint8_t* st = smem + s * L::kStage;
          if (k < n_main) {
            mbar_arrive_expect_tx(&full[s], L::kA + L::kB);
#pragma unroll
            for (int h = 0; h < kBM / kActBoxRows; ++h)
              tma_load_2d(st + h * kActBoxRows * kBK, &maps.a, &full[s], k * kBK, m0 + h * kActBoxRows);
#pragma unroll
            for (int h = 0; h < kBN / kWeightBoxRows; ++h)
              tma_load_2d(st + L::kA + h * kWeightBoxRows * kBK, &maps.b, &full[s], k * kBK, n0 + h * kWeightBoxRows);
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
        for (int j = max(0, gs - kSwSlots); j < gs; ++j)
          mbar_wait(&sw_full[j % kSwSlots], (j / kSwSlots) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_q = idesc_dense(kFmtF32, kFmtE4M3, kFmtE4M3, kBM, kBN);
    const uint32_t idesc_lr = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, kBM, kBN);
    bool ok = true;
    int it = 0;  // k-tiles consumed
    int ga = 0;  // accumulations started (groups and branch passes) over all tiles
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      for (int k = 0; k < n_main + n_lr && ok; ++k, ++it) {
        const int s = it % kStages;
        const bool main_tile = k < n_main;
        if (!main_tile && k == n_main) {
          // the branch accumulates all its k-tiles into one buffer
          ok = mbar_wait(&d_empty[ga % kDBufs], ((ga / kDBufs) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
        }
        ok = mbar_wait(&full[s], (it / kStages) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * L::kStage);
        const uint32_t b_base = a_base + L::kA;
        if (main_tile) {
          for (int gg = 0; gg < 2 && ok; ++gg, ++ga) {
            ok = mbar_wait(&d_empty[ga % kDBufs], ((ga / kDBufs) & 1) ^ 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {  // one fixed thread issues every tcgen05 op, so its commits track them all
              const uint32_t d = tmem + (ga % kDBufs) * kBN;
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint64_t ad = smem_desc(a_base + 64 * gg + 32 * j, 16, 1024, kSw128);
                const uint64_t bd = smem_desc(b_base + 64 * gg + 32 * j, 16, 1024, kSw128);
                mma_f8f6f4(d, ad, bd, idesc_q, j);
              }
              tc_commit(&d_full[ga % kDBufs]);
            }
            __syncwarp();
          }
          if (!ok) break;
        } else {
          if (lane == 0) {
            const uint32_t d = tmem + (ga % kDBufs) * kBN;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint64_t ad = smem_desc(a_base + 32 * j, 16, 512, kSw64);
              const uint64_t bd = smem_desc(b_base + 32 * j, 16, 512, kSw64);
              mma_f16(d, ad, bd, idesc_lr, (k > n_main || j > 0) ? 1u : 0u);
            }
            if (k == n_main + n_lr - 1) tc_commit(&d_full[ga % kDBufs]);
          }
          __syncwarp();
          if (k == n_main + n_lr - 1) ++ga;
        }
        if (lane == 0) tc_commit(&empty[s]);
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ drain / epilogue
    const int dw = warp - kFirstDrainWarp;  // drain warp 0..15
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int col0 = (dw >> 2) * kCols;     // this warp's slice of the tile's columns
    bool ok = true;
    int ga = 0;  // accumulations drained
    int gs = 0;  // scale vectors consumed
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int m0 = (tile / n_blocks) * kBM, n0 = (tile % n_blocks) * kBN;
      const int row = m0 + 32 * q + lane;
      float2 acc[kCols / 2];
#pragma unroll
      for (int j = 0; j < kCols / 2; ++j) acc[j] = make_float2(0.f, 0.f);
      // the groups, then (with a branch) one pass for the low-rank product
      const int n_acc = n_groups + (n_lr > 0 ? 1 : 0);
      for (int g = 0; g < n_acc && ok; ++g, ++ga) {
        const bool branch = (g == n_groups);
        const int ws = gs % kSwSlots;
        if (!branch) {
          ok = mbar_wait(&sw_full[ws], (gs / kSwSlots) & 1, abort_flag, p.status);
          if (!ok) break;
        }
        ok = mbar_wait(&d_full[ga % kDBufs], (ga / kDBufs) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + (ga % kDBufs) * kBN + col0 + (static_cast<uint32_t>(32 * q) << 16);
        const float* slot = sw_ring + ws * (kBN + kBM);
        const float sx = branch ? 1.f : slot[kBN + 32 * q + lane];
        const float2 sx2 = make_float2(sx, sx);
        const float4* sw4 = reinterpret_cast<const float4*>(slot + col0);
        // TMEM loads of 8 columns: 8 accumulator registers per load keep the
        // drain warp within the register budget of an 18-warp CTA.
        constexpr int kNC = kCols / 8;
#pragma unroll
        for (int c = 0; c < kNC; ++c) {
          uint32_t r[8];
          tmem_ld8(d + 8 * c, r);
          tmem_ld_wait();
          if (c == kNC - 1) {
            // every load of this group has landed: the accumulator is free
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[ga % kDBufs]);
          }
          if (branch) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              acc[4 * c + j] = __fadd2_rn(acc[4 * c + j], make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])));
          } else {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float4 w = sw4[2 * c + j];
              const float2 w01 = __fmul2_rn(sx2, make_float2(w.x, w.y));
              const float2 w23 = __fmul2_rn(sx2, make_float2(w.z, w.w));
              float2& a01 = acc[4 * c + 2 * j];
              float2& a23 = acc[4 * c + 2 * j + 1];
              a01 = __ffma2_rn(w01, make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])), a01);
              a23 = __ffma2_rn(w23, make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])), a23);
            }
          }
        }
        if (!branch) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&sw_empty[ws]);
          ++gs;
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


cudaError_t launch_gemm_int4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemI4::kTotal);
  });
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int n_tiles = (p.M_pad / kBM) * ((p.N + kBN - 1) / kBN);
  const int grid = n_tiles < sms ? n_tiles : sms;
  gemm_int4_kernel<<<grid, kThreads, SmemI4::kTotal, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace svdq
