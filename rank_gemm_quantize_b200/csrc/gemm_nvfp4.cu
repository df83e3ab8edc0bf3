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
// Two SMs work as one (a cluster of two CTAs, tcgen05 .cta_group::2): the
// pair computes a 256 x 256 output tile with M = 256 MMAs. Each CTA loads
// only its own 128 rows of the activation codes and its own 128 columns of the
// weight codes (plain TMA, no multicast), plus its rows' activation scale
// factors and the weight scale factors of all 256 columns; the tensor cores
// of the pair read both CTAs' halves. Per SM that is 38 KB of operands per
// 256-deep k-tile instead of 54 KB for a 128 x 256 tile on one SM.
//
// Persistent kernel, one pair per two SMs. Warp roles (19 warps per CTA):
//   warp 0  producer (both CTAs): per tile its bias slice (bulk copy, local
//           ring), then the k-tiles: A and B codes and both scale-factor
//           tiles by TMA, completing on the leader CTA's stage barrier;
//           then the branch k-tiles (32-column slices of T' and L2^T);
//   warp 18 scale factors (leader): copies each stage's scale factors of both
//           CTAs into their TMEM (tcgen05.cp .cta_group::2) and commits;
//   warp 1  TMEM owner (both) and MMA issuer (leader, one thread): per k-tile
//           4 block-scaled MMAs, per branch k-tile 2 kind::f16 MMAs; the
//           commits free the stage in both CTAs and mark the tile;
//   warps 2-17 epilogue (both), four per TMEM lane quarter (enough warps to
//           hide the latency of the MLP variant's per-element work): each
//           reads its 32 rows x 64 columns of its CTA's accumulator 32
//           columns at a time, scales, adds the bias and packs bf16; after
//           the last TMEM load it tells the leader that TMEM is free (the
//           next tile's MMAs start). Each 32 x 32 chunk goes through the
//           warp's one 2 KB staging box (64-byte swizzle) and out with a TMA
//           store (rows and columns past M and N are clipped by the tensor
//           map); the small staging leaves shared memory for a fifth stage.
//
// MLP-block variant (kMlp, the up layer of up -> GELU -> down): the branch
// reads T as a bf16 pair (T + T_lo, about 16 significant bits), so the up
// output, and with it the bf16 rounding of its GELU that decides the down
// layer's codes, matches the exact product far more closely. The epilogue
// does not store Y. It rounds the output to bf16, applies GELU (erf form,
// float32) and rounds to bf16 (h: the tensor a plain composition of the two
// layers would pass on), then smooths and NVFP4-quantizes h for the down
// layer into that layer's code and scale buffers, and stages h in shared
// memory. The leader then contracts the staged h with the down layer's
// 1/s-folded factor (L1s^T slices loaded per tile) into a TMEM accumulator:
// the down layer's branch input T. A pair takes a contiguous range of tiles
// in row-major tile order, so T accumulates over the pair's tiles of one
// 256-row block; it is flushed as a float partial when the row block changes
// and the partials are summed in a fixed order by mlp_t_reduce_kernel. The
// contraction of tile i is issued after the next tile's mainloop MMAs, so it
// overlaps the epilogue instead of waiting for it.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int kBM = 128;       // rows per CTA (the pair covers 256)
constexpr int kBN = 256;       // columns per pair tile
constexpr int kBNHalf = 128;   // weight rows each CTA loads
constexpr int kBKBytes = 128;  // 256 E2M1 values per row per k-tile
constexpr int kEpiWarps = 16;                   // four per TMEM lane quarter
constexpr int kEpiCols = kBN / (kEpiWarps / 4);  // columns of the tile each epilogue warp takes (64)
constexpr int kCpWarp = 2 + kEpiWarps;  // copies scale factors into TMEM
constexpr int kThreads = (3 + kEpiWarps) * 32;

template <bool kMlp>
struct SmemNv {
  static constexpr int kStages = kMlp ? 3 : 5;
  static constexpr int kA = kBM * kBKBytes;       // 16 KB
  static constexpr int kB = kBNHalf * kBKBytes;   // 16 KB
  static constexpr int kSfa = 4 * 512;            // this CTA's 128 rows, 4 k-blocks of 64
  static constexpr int kSfb = (kBN / 128) * 4 * 512;  // all 256 columns, 4 k-blocks
  static constexpr int kStage = kA + kB + kSfa + kSfb;  // 38 KB
  static constexpr int kBiasOff = kStages * kStage;
  static constexpr int kBias = kBN * 2;           // bf16 bias slice of a tile
  // Y staging for the TMA stores (16 warps x one 32 x 64 box); in the MLP
  // variant the same 64 KB hold h as four K-major 128 x 64 bf16 chunks.
  static constexpr int kStgOff = kBiasOff + 2 * kBias;
  // Y staging (plain): one 32 x 32 box per epilogue warp (2 KB, 64-byte swizzle), reused
  // chunk after chunk; in the MLP variant the 64 KB hold h as four K-major 128 x 64 chunks.
  static constexpr int kStgWarp = 32 * 64;
  static constexpr int kStg = kMlp ? 4 * kBM * 128 : kEpiWarps * kStgWarp;  // 64 KB / 32 KB
  static constexpr int kHChunk = kBM * 128;          // 16 KB: 128 rows x 64 bf16
  static constexpr int kIsOff = kStgOff + kStg;      // MLP: down-layer inv_s slices, 2 x 256 floats
  static constexpr int kIs = kMlp ? kBN * 4 : 0;
  static constexpr int kL1Off = kIsOff + 2 * kIs;    // MLP: down-layer L1s^T slices, 2 slots
  static constexpr int kL1Part = (kMlpDownRP / 2) * 128;  // this CTA's 16 rows x 64 bf16 (hi or lo)
  static constexpr int kL1Slot = kMlp ? 4 * 2 * kL1Part : 0;  // 4 chunks x (hi, lo)
  static constexpr int kBarOff = kL1Off + 2 * kL1Slot;
  static constexpr int kTotal = kBarOff + 512 + 1024;
};
static_assert(SmemNv<false>::kTotal <= 232448 && SmemNv<true>::kTotal <= 232448, "shared memory budget");
static_assert(SmemNv<false>::kStage % 1024 == 0 && SmemNv<true>::kStgOff % 1024 == 0 &&
                  SmemNv<false>::kStgOff % 1024 == 0 && SmemNv<true>::kL1Off % 1024 == 0,
              "swizzled tiles start 1 KB-aligned");
static_assert(2 * kBM * 64 <= SmemNv<true>::kA, "T and its low part share a stage's A slot");
static_assert(kBNHalf == kWeightBoxRows && kBM == kActBoxRows, "each CTA loads one box per operand");

// TMEM columns (each CTA): accumulator [0, 256), then one scale-factor slot per
// shared-memory stage (A: 16 columns, B: 32), so copying the next k-tile's
// scale factors never waits for the MMAs still reading the previous ones;
// then (MLP) the down layer's T accumulator (64 columns: the products with the
// factor's high and low bf16 parts side by side, summed when read out).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfSlotCols = 16 + 2 * 16;
constexpr uint32_t kSfaCol = kBN;
constexpr uint32_t kSfbCol = kBN + 16;
template <bool kMlp>
constexpr uint32_t t_acc_col() { return kBN + SmemNv<kMlp>::kStages * kSfSlotCols; }
static_assert(t_acc_col<true>() + 2 * kMlpDownRP <= kTmemCols && t_acc_col<false>() <= kTmemCols, "TMEM budget");

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// GELU(y) = y Phi(y) = y (1 + erf(y / sqrt 2)) / 2 of a packed bf16 pair,
// returned as the packed bf16 pair of the results. With x = |y| / sqrt 2,
// (1 + erf(y / sqrt 2)) / 2 is 1 - erfc(x) / 2 for y >= 0 and erfc(x) / 2 for
// y < 0 (no cancellation on the negative side), and
//   erfc(x) / 2 = 2^(-u^2) q(u),  u = |y| sqrt(log2(e) / 2),
// where q(u) = erfcx(x) / 2 is approximated on [0, 6 sqrt(log2 e)] by a
// degree-10 polynomial whose coefficients were fitted here by weighted
// minimax (Lawson's iteration) with weight 2^(-u^2), so that the fit's error
// is measured on erfc itself: at most 2.7e-7 absolute in float32 (u is
// clamped at the end of that range, where erfc < 3e-17). Both values go
// through packed float32 arithmetic (two per instruction); one ex2 each.
__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint32_t gelu_bf16x2(uint32_t w) {
  const float2 y = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  const uint32_t a = w & 0x7FFF7FFFu;  // |y|
  float2 u = __fmul2_rn(make_float2(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u)),
                        make_float2(8.493217826e-01f, 8.493217826e-01f));
  u.x = fminf(u.x, 7.206734657e+00f);
  u.y = fminf(u.y, 7.206734657e+00f);
  const float2 uu = __fmul2_rn(u, u);
  float2 q = make_float2(8.354404599e-06f, 8.354404599e-06f);
  q = __ffma2_rn(q, u, make_float2(-1.531047310e-04f, -1.531047310e-04f));
  q = __ffma2_rn(q, u, make_float2(1.254777540e-03f, 1.254777540e-03f));
  q = __ffma2_rn(q, u, make_float2(-6.194117013e-03f, -6.194117013e-03f));
  q = __ffma2_rn(q, u, make_float2(2.115210705e-02f, 2.115210705e-02f));
  q = __ffma2_rn(q, u, make_float2(-5.501661450e-02f, -5.501661450e-02f));
  q = __ffma2_rn(q, u, make_float2(1.175282001e-01f, 1.175282001e-01f));
  q = __ffma2_rn(q, u, make_float2(-2.162939161e-01f, -2.162939161e-01f));
  q = __ffma2_rn(q, u, make_float2(3.464582562e-01f, 3.464582562e-01f));
  q = __ffma2_rn(q, u, make_float2(-4.697118402e-01f, -4.697118402e-01f));
  q = __ffma2_rn(q, u, make_float2(4.999999404e-01f, 4.999999404e-01f));
  const float2 hc = __fmul2_rn(make_float2(ex2_approx(-uu.x), ex2_approx(-uu.y)), q);  // erfc(x) / 2
  // 1 - erfc/2 for y >= 0 (sign bit clear), erfc/2 itself for y < 0
  const float2 om = __ffma2_rn(hc, make_float2(-1.f, -1.f), make_float2(1.f, 1.f));
  const float2 t = make_float2((w & 0x8000u) ? hc.x : om.x, (w & 0x80000000u) ? hc.y : om.y);
  const float2 g = __fmul2_rn(y, t);
  return pack_bf16x2(g.x, g.y);
}

// The tile range of pair `pair`: round-robin for the plain GEMM (the pairs in
// flight share the weight panel in L2); contiguous in row-major tile order for
// the MLP variant (the down layer's T accumulates over a row block).
struct TileRange {
  int first, last, step;
};
template <bool kMlp>
__device__ __forceinline__ TileRange tile_range(int pair, int n_pairs, int n_tiles) {
  if (kMlp) {
    return {static_cast<int>((static_cast<long long>(pair) * n_tiles) / n_pairs),
            static_cast<int>((static_cast<long long>(pair + 1) * n_tiles) / n_pairs), 1};
  }
  return {pair, n_tiles, n_pairs};
}

// Pair p takes tiles [floor(p T / P), floor((p + 1) T / P)) of the T tiles
// (P <= T pairs, so no range is empty). The pair holding tile t is the
// smallest p with floor((p + 1) T / P) > t, i.e. p = ceil((t + 1) P / T) - 1.
// The host keeps T P below 2^31, so the products fit in 32 bits.
__host__ __device__ inline int mlp_pair_of_tile(int t, int n_tiles, int n_pairs) {
  const int p = ((t + 1) * n_pairs + n_tiles - 1) / n_tiles - 1;
  return p < 0 ? 0 : (p > n_pairs - 1 ? n_pairs - 1 : p);
}
// The first pair whose range holds a tile of 256-row block mp.
__host__ __device__ inline int mlp_first_pair(int mp, int n_blocks, int n_tiles, int n_pairs) {
  return mlp_pair_of_tile(mp * n_blocks, n_tiles, n_pairs);
}
// The number of pairs whose ranges hold tiles of row block mp (the partial
// slots it uses): from the pair of its first tile to the pair of its last.
__host__ __device__ inline int mlp_block_pairs(int mp, int n_blocks, int n_tiles, int n_pairs) {
  return mlp_pair_of_tile(mp * n_blocks + n_blocks - 1, n_tiles, n_pairs) -
         mlp_pair_of_tile(mp * n_blocks, n_tiles, n_pairs) + 1;
}

template <bool kMlp>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const GemmParams p, const MlpDownParams mlp, const __grid_constant__ GemmMaps maps) {
  using L = SmemNv<kMlp>;
  constexpr int kStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);  // [kStages] (leader) both CTAs' loads landed
  uint64_t* empty = full + kStages;      // [kStages] (both) the MMAs are done with the stage
  uint64_t* acc_full = empty + kStages;  // (both) the tile's accumulator is complete
  uint64_t* acc_empty = acc_full + 1;    // (leader) both CTAs' epilogues copied the accumulator out
  uint64_t* bias_full = acc_empty + 1;   // [2] (both, local)
  uint64_t* bias_empty = bias_full + 2;  // [2] (both, local)
  uint64_t* drain = bias_empty + 2;      // (both) every MMA has completed
  uint64_t* sf_ready = drain + 1;        // [kStages] (leader) scale factors of the stage are in TMEM
  uint64_t* cp_done = sf_ready + kStages;
  // MLP block only:
  uint64_t* is_full = cp_done + 1;       // [2] (both, local) down-layer inv_s slice landed
  uint64_t* is_empty = is_full + 2;      // [2] (both, local)
  uint64_t* l1_full = is_empty + 2;      // [2] (leader) both CTAs' L1s^T slices landed
  uint64_t* l1_empty = l1_full + 2;      // [2] (both) the T MMAs of the slot's tile completed
  uint64_t* h_ready = l1_empty + 2;      // (leader) both CTAs staged the tile's h
  uint64_t* t_full = h_ready + 1;        // (both) T accumulator holds a finished row-block partial
  uint64_t* t_empty = t_full + 1;        // (leader) both CTAs read that partial out
  uint64_t* sf_full = t_empty + 1;       // [kStages] (leader) both CTAs' scale-factor tiles of the stage landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_full + kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int n_blocks = p.N_pad / kBN;
  const int m_pairs = (p.M_pad + 2 * kBM - 1) / (2 * kBM);
  const int n_tiles = m_pairs * n_blocks;
  const int kb_total = p.K / 64;
  const int n_main = (p.K + 255) / 256;
  const int n_lr = p.RP / 32;
  const int n_items = n_main + n_lr;
  const TileRange tr = tile_range<kMlp>(pair, n_pairs, n_tiles);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
      mbar_init(&sf_full[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bias_full[b], 1);
      mbar_init(&bias_empty[b], kEpiWarps);
      mbar_init(&is_full[b], 1);
      mbar_init(&is_empty[b], kEpiWarps);
      mbar_init(&l1_full[b], 1);
      mbar_init(&l1_empty[b], 1);
    }
    mbar_init(drain, 1);
    mbar_init(cp_done, 1);
    mbar_init(h_ready, 2 * kEpiWarps);
    mbar_init(t_full, 1);
    mbar_init(t_empty, 2 * 4);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      prefetch_tensormap(&maps.a);
      prefetch_tensormap(&maps.b);
      prefetch_tensormap(&maps.sfa);
      prefetch_tensormap(&maps.sfb);
      if (n_lr > 0) {  // no branch (rank 0): its maps are never read
        prefetch_tensormap(&maps.t);
        prefetch_tensormap(&maps.l2);
      }
      if (kMlp) {
        prefetch_tensormap(&maps.l1h_down);
        prefetch_tensormap(&maps.l1l_down);
        if (n_lr > 0) prefetch_tensormap(&maps.t_lo);
      }
      bool ok = true;
      int it = 0;          // k-tiles issued over all tiles of this CTA
      int ti = 0;          // tiles of this CTA
      int last_bias = -1;  // last tile whose local copies were issued
      for (int tile = tr.first; tile < tr.last && ok; tile += tr.step, ++ti) {
        const int mp = tile / n_blocks, nb = tile % n_blocks;
        const int m0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;  // this CTA's rows
        const int n0 = nb * kBN;
        const int bs = ti & 1;
        ok = mbar_wait(&bias_empty[bs], ((ti >> 1) & 1) ^ 1, abort_flag, p.status);
        if (ok && kMlp) ok = mbar_wait(&is_empty[bs], ((ti >> 1) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        mbar_arrive_expect_tx(&bias_full[bs], L::kBias);
        bulk_load(smem + L::kBiasOff + bs * L::kBias, p.bias + n0, L::kBias, &bias_full[bs]);
        if (kMlp) {
          mbar_arrive_expect_tx(&is_full[bs], L::kIs);
          bulk_load(smem + L::kIsOff + bs * L::kIs, mlp.inv_s + n0, L::kIs, &is_full[bs]);
        }
        last_bias = ti;
        for (int k = 0; k < n_items && ok; ++k, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          uint8_t* st = smem + s * L::kStage;
          const uint32_t fb = leader_addr(&full[s]);
          if (k < n_main) {
            // the scale factors first, on their own barrier: their copies into TMEM overlap the
            // landing of the codes instead of following it
            const uint32_t sb = leader_addr(&sf_full[s]);
            if (leader) {
              mbar_arrive_expect_tx(&sf_full[s], 2 * (L::kSfa + L::kSfb));
              mbar_arrive_expect_tx(&full[s], 2 * (L::kA + L::kB));
            }
            const int kb0 = k * 4;
            // scale-factor atoms (512 bytes each): 4 k-blocks of this CTA's row block, and of both column blocks
            tma_load_2d_pair(st + L::kA + L::kB, &maps.sfa, sb, 0, (m0 / 128) * kb_total + kb0);
#pragma unroll
            for (int h = 0; h < kBN / 128; ++h)
              tma_load_2d_pair(st + L::kA + L::kB + L::kSfa + h * 2048, &maps.sfb, sb, 0,
                               (nb * (kBN / 128) + h) * kb_total + kb0);
            tma_load_2d_pair(st, &maps.a, fb, k * kBKBytes, m0);
            tma_load_2d_pair(st + L::kA, &maps.b, fb, k * kBKBytes, n0 + static_cast<int>(rank) * kBNHalf);
          } else {
            if (leader) {
              mbar_arrive(&sf_full[s]);  // no scale factors in a branch k-tile
              mbar_arrive_expect_tx(&full[s], 2 * ((kMlp ? 2 : 1) * kBM * 64 + kBNHalf * 64));
            }
            const int c = k - n_main;  // 32-column slice of the branch
            tma_load_2d_pair(st, &maps.t, fb, c * 32, m0);
            if (kMlp) tma_load_2d_pair(st + kBM * 64, &maps.t_lo, fb, c * 32, m0);
            tma_load_2d_pair(st + L::kA, &maps.l2, fb, c * 32, n0 + static_cast<int>(rank) * kBNHalf);
          }
        }
        if (kMlp && ok) {
          // this CTA's half of the down layer's factor rows for the tile's four 64-wide K chunks. It is
          // used by the tile's T contraction, which comes after the next tile's mainloop, so it is
          // loaded after this tile's k-tiles: waiting for the slot (freed by the contraction of the
          // tile two back) never delays a k-tile.
          ok = mbar_wait(&l1_empty[bs], ((ti >> 1) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          const uint32_t lb = leader_addr(&l1_full[bs]);
          if (leader) mbar_arrive_expect_tx(&l1_full[bs], 2 * L::kL1Slot);
          uint8_t* l1 = smem + L::kL1Off + bs * L::kL1Slot;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int y = static_cast<int>(rank) * (kMlpDownRP / 2);
            tma_load_2d_pair(l1 + (2 * c) * L::kL1Part, &maps.l1h_down, lb, n0 + 64 * c, y);
            tma_load_2d_pair(l1 + (2 * c + 1) * L::kL1Part, &maps.l1l_down, lb, n0 + 64 * c, y);
          }
        }
      }
      if (!ok) {
        // gave up: let this CTA's local copies in flight land before it exits
        volatile int no_abort = 0;
        for (int t2 = last_bias - 1; t2 <= last_bias; ++t2)
          if (t2 >= 0) {
            mbar_wait(&bias_full[t2 & 1], (t2 >> 1) & 1, &no_abort, nullptr);
            if (kMlp) mbar_wait(&is_full[t2 & 1], (t2 >> 1) & 1, &no_abort, nullptr);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader) {
      const uint32_t idesc_main = idesc_block_scaled(2 * kBM, kBN);
      const uint32_t idesc_lr = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, 2 * kBM, kBN);
      // T contraction: N = 64, each CTA's 32 B rows being its 16 ranks of L1s^T's high part, then
      // the same 16 ranks' low part (adjacent in the slot), so one MMA takes both
      const uint32_t idesc_t = idesc_dense(kFmtF32, kFmtBF16, kFmtBF16, 2 * kBM, 2 * kMlpDownRP);
      bool ok = true;
      int it = 0, ti = 0;
      int flushes = 0;  // MLP: row-block partials of T flushed so far
      // MLP: the down layer's T contraction of tile j (issued after tile j+1's mainloop)
      auto issue_t = [&](int j, int tile_j) -> bool {
        const int mp = tile_j / n_blocks;
        const bool first = tile_j == tr.first || (tile_j - 1) / n_blocks != mp;
        const bool last = tile_j + 1 == tr.last || (tile_j + 1) / n_blocks != mp;
        if (first && flushes > 0 && !mbar_wait(t_empty, (flushes - 1) & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(&l1_full[j & 1], (j >> 1) & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(h_ready, j & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t hst = smem_u32(smem + L::kStgOff);
          const uint32_t l1 = smem_u32(smem + L::kL1Off + (j & 1) * L::kL1Slot);
          const uint32_t tacc = tmem + t_acc_col<kMlp>();
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16_pair(tacc, smem_desc(hst + c * L::kHChunk + 32 * ks, 16, 1024, kSw128),
                           smem_desc(l1 + (2 * c) * L::kL1Part + 32 * ks, 16, 1024, kSw128), idesc_t,
                           (first && c == 0 && ks == 0) ? 0u : 1u);
          tc_commit_pair_mc(&l1_empty[j & 1], 0x3);
          if (last) tc_commit_pair_mc(t_full, 0x3);
        }
        __syncwarp();
        if (last) ++flushes;
        return true;
      };
      int prev_tile = -1;
      for (int tile = tr.first; tile < tr.last && ok; tile += tr.step, ++ti) {
        // both CTAs' epilogues have copied the previous tile's accumulator out of TMEM
        ok = mbar_wait(acc_empty, (ti & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        for (int k = 0; k < n_items && ok; ++k, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&full[s], (it / kStages) & 1, abort_flag, p.status) &&
               mbar_wait(&sf_ready[s], (it / kStages) & 1, abort_flag, p.status);
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
                mma_nvf4_pair(tmem, ad, bd, idesc_main, t_sfa + 4 * j, t_sfb + (kBN / 32) * j,
                              (k > 0 || j > 0) ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint64_t ad = smem_desc(a_base + 32 * j, 16, 512, kSw64);
                const uint64_t bd = smem_desc(b_base + 32 * j, 16, 512, kSw64);
                mma_f16_pair(tmem, ad, bd, idesc_lr, 1u);
                if (kMlp)  // T's low part: the block's GELU input carries about 16 bits of T
                  mma_f16_pair(tmem, smem_desc(a_base + kBM * 64 + 32 * j, 16, 512, kSw64), bd, idesc_lr, 1u);
              }
            }
            tc_commit_pair_mc(&empty[s], 0x3);  // the stage is free in both CTAs
          }
          __syncwarp();
        }
        if (!ok) break;
        if (kMlp && ti > 0) {
          ok = issue_t(ti - 1, prev_tile);
          if (!ok) break;
        }
        if (lane == 0) tc_commit_pair_mc(acc_full, 0x3);  // also implies the T contraction above completed
        __syncwarp();
        prev_tile = tile;
      }
      if (kMlp && ok && ti > 0) issue_t(ti - 1, prev_tile);
    }
  } else if (warp == kCpWarp) {
    // ------------------------------------------------------------ scale factors to TMEM (leader)
    // One stage ahead of the MMA thread at most (it waits for each stage's
    // copies): the copies and the MMAs come from different threads.
    if (leader && lane == 0) {
      bool ok = true;
      int it = 0;
      for (int tile = tr.first; tile < tr.last && ok; tile += tr.step) {
        for (int k = 0; k < n_items && ok; ++k, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(&sf_full[s], (it / kStages) & 1, abort_flag, p.status);
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
              tmem_cp_32x128b_x4_pair(t_sfa + 4 * j, smem_desc(sfa_base + 512 * j, 16, 128, kSwNone));
#pragma unroll
              for (int h = 0; h < kBN / 128; ++h)
                tmem_cp_32x128b_x4_pair(t_sfb + (kBN / 32) * j + 4 * h,
                                        smem_desc(sfb_base + h * 2048 + 512 * j, 16, 128, kSwNone));
            }
          }
          tc_commit_pair(smem_u32(&sf_ready[s]));
        }
      }
      tc_commit_pair(smem_u32(cp_done));  // arrives once every copy issued above has finished
      volatile int no_abort = 0;
      mbar_wait(cp_done, 0, &no_abort, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;                  // 0..7
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int col0 = (ew >> 2) * kEpiCols;    // this warp's columns of the tile
    const int rc = 32 * q + lane;             // this thread's row within the CTA's 128
    uint8_t* stg = smem + L::kStgOff + ew * L::kStgWarp;
    bool ok = true;
    int ti = 0;
    int flushes = 0;
    // MLP: the pair's T partial of the row block that ended with tile_j -> workspace
    auto flush_t = [&](int tile_j) -> bool {
      if (!mbar_wait(t_full, flushes & 1, abort_flag, p.status)) return false;
      ++flushes;
      if (ew >= 4) return true;  // one warp per TMEM lane quarter reads the partial
      tc_fence_after();
      const int mp = tile_j / n_blocks;
      const int slot = pair - mlp_first_pair(mp, n_blocks, n_tiles, n_pairs);
      float* dst = mlp.tpart + ((static_cast<size_t>(mp) * mlp.slots + slot) * (2 * kBM) +
                                static_cast<int>(rank) * kBM + rc) * kMlpDownRP;
      // accumulator columns: [16 ranks high | the same ranks low] per CTA half of the pair
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + t_acc_col<kMlp>() + 32 * half, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(dst + 16 * half + e) =
              make_float4(__uint_as_float(r[e]) + __uint_as_float(r[e + 16]),
                          __uint_as_float(r[e + 1]) + __uint_as_float(r[e + 17]),
                          __uint_as_float(r[e + 2]) + __uint_as_float(r[e + 18]),
                          __uint_as_float(r[e + 3]) + __uint_as_float(r[e + 19]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(t_empty, 0);
      return true;
    };
    int prev_tile = -1;
    for (int tile = tr.first; tile < tr.last && ok; tile += tr.step, ++ti) {
      const int mp = tile / n_blocks, nb = tile % n_blocks;
      const int row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM + 32 * q;  // first row of this warp
      const int bs = ti & 1;
      ok = mbar_wait(&bias_full[bs], (ti >> 1) & 1, abort_flag, p.status);
      if (ok && kMlp) ok = mbar_wait(&is_full[bs], (ti >> 1) & 1, abort_flag, p.status);
      if (ok) ok = mbar_wait(acc_full, ti & 1, abort_flag, p.status);
      if (!ok) break;
      tc_fence_after();
      const uint4* bias4 = reinterpret_cast<const uint4*>(smem + L::kBiasOff + bs * L::kBias) + col0 / 8;
      const uint32_t ta = tmem + (static_cast<uint32_t>(32 * q) << 16) + col0;
      // Phase A: the accumulator -> y = out_scale acc + b, bf16. Plain: into this warp's 32 x 32
      // staging box and out with a TMA store, 32 columns at a time; MLP block: into the K-major
      // h chunks, where phase B turns y into h in place.
#pragma unroll
      for (int c = 0; c < kEpiCols / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(ta + 32 * c, r);
        tmem_ld_wait();
        uint32_t o[16];  // this thread's 32 values of the chunk as packed bf16
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 bw = bias4[4 * c + v];
          const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 yv = __ffma2_rn(make_float2(__uint_as_float(r[8 * v + 2 * e]), __uint_as_float(r[8 * v + 2 * e + 1])),
                                         make_float2(p.out_scale, p.out_scale),
                                         make_float2(__uint_as_float(bb[e] << 16), __uint_as_float(bb[e] & 0xFFFF0000u)));
            o[4 * v + e] = pack_bf16x2(yv.x, yv.y);
          }
        }
        if (c == kEpiCols / 32 - 1) {
          // every load of the tile has landed: this CTA's share of TMEM is free, the next tile's
          // MMAs start; the bias slot is free too
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster(acc_empty, 0);
            mbar_arrive(&bias_empty[bs]);
          }
        }
        if (!kMlp) {
          if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read the box
          __syncwarp();
          uint8_t* row = stg + lane * 64;  // 64-byte rows, 16-byte chunk j at j ^ ((row / 2) % 4)
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(row + ((v ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&maps.y, stg, nb * kBN + col0 + 32 * c, row0);
            bulk_commit_group();
          }
        } else {
          const int cn = col0 + 32 * c;
          uint8_t* row = smem + L::kStgOff + (cn >> 6) * L::kHChunk + rc * 128;
          const int chunk0 = (cn & 63) >> 3;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(row + (((chunk0 + v) ^ (rc & 7)) << 4)) =
                make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
      }
      if (kMlp) {
        // Phase B, overlapping the next tile's mainloop. B1: h = bf16(GELU(y)) in place over this
        // thread's row slice; then the T contraction may read h (the fence comes before any of this
        // tile's global stores, so it does not wait for them). B2: the down layer's smoothing and
        // NVFP4 groups of 16 from the staged h.
        const float* is_tile = reinterpret_cast<const float*>(smem + L::kIsOff + bs * L::kIs);
        const int m = row0 + lane;
        uint8_t* hrow = smem + L::kStgOff + (col0 >> 6) * L::kHChunk + rc * 128;
#pragma unroll
        for (int piece = 0; piece < kEpiCols / 64; ++piece) {
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {  // 16-byte chunk of the 128-byte row (8 values)
            uint4* pc = reinterpret_cast<uint4*>(hrow + piece * L::kHChunk + ((c16 ^ (rc & 7)) << 4));
            const uint4 u = *pc;
            *pc = make_uint4(gelu_bf16x2(u.x), gelu_bf16x2(u.y), gelu_bf16x2(u.z), gelu_bf16x2(u.w));
          }
        }
        fence_proxy_async_smem();  // h is read by the T contraction's MMAs
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(h_ready, 0);
#pragma unroll 1
        for (int piece = 0; piece < kEpiCols / 64; ++piece) {
          const int cn = col0 + 64 * piece;  // first column of the 64 within the tile
          const uint8_t* row = hrow + piece * L::kHChunk;
          uint32_t cw[8];
          uint32_t sbw = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint4 u0 = *reinterpret_cast<const uint4*>(row + (((2 * g) ^ (rc & 7)) << 4));
            const uint4 u1 = *reinterpret_cast<const uint4*>(row + (((2 * g + 1) ^ (rc & 7)) << 4));
            const uint32_t hw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float v[16];
            const float* is = is_tile + cn + 16 * g;
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 s4 = *reinterpret_cast<const float4*>(is + e);
              const float2 a = __fmul2_rn(make_float2(__uint_as_float(hw[e / 2] << 16),
                                                      __uint_as_float(hw[e / 2] & 0xFFFF0000u)),
                                          make_float2(s4.x, s4.y));
              const float2 b2 = __fmul2_rn(make_float2(__uint_as_float(hw[e / 2 + 1] << 16),
                                                       __uint_as_float(hw[e / 2 + 1] & 0xFFFF0000u)),
                                           make_float2(s4.z, s4.w));
              v[e] = a.x;
              v[e + 1] = a.y;
              v[e + 2] = b2.x;
              v[e + 3] = b2.y;
            }
            sbw |= nvfp4_quant16(v, mlp.denom, mlp.g_x, cw[2 * g], cw[2 * g + 1]) << (8 * g);
          }
          if (m < mlp.M_pad) {
            const int n = nb * kBN + cn;  // column of the up output = k of the down layer
            uint4* dst = reinterpret_cast<uint4*>(mlp.codes + static_cast<size_t>(m) * (mlp.K >> 1) + (n >> 1));
            dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
            // scale-factor atom (m / 128) * (K / 64) + n / 64 holds the four groups as adjacent bytes
            const size_t atom = static_cast<size_t>(m >> 7) * (mlp.K >> 6) + (n >> 6);
            *reinterpret_cast<uint32_t*>(mlp.scales + atom * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4) = sbw;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&is_empty[bs]);
      }
      // MLP: the previous tile closed a row block: its partial is complete (its
      // contraction was committed before this tile's accumulator)
      if (kMlp && prev_tile >= 0 && (prev_tile / n_blocks) != mp) {
        ok = flush_t(prev_tile);
        if (!ok) break;
      }
      prev_tile = tile;
    }
    if (kMlp && ok && prev_tile >= 0) flush_t(prev_tile);
    if (!kMlp) {
      if (lane == 0) bulk_wait_group<0>();  // every store of this warp has completed
      __syncwarp();
    }
  }

  // ------------------------------------------------------------ teardown
  // The leader's last commit tells both CTAs that every MMA has completed;
  // the cluster barrier keeps each CTA alive until its partner is done
  // signalling its barriers, then both free the pair's TMEM.
  if (warp == 1 && leader && lane == 0) tc_commit_pair_mc(drain, 0x3);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort, nullptr);
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// T = bf16(t_scale * sum over the partial slots of each 256-row block, in slot
// order); one thread per element, 8 rows per CTA.
constexpr int kReduceRows = 8;
constexpr int kReduceUnroll = 8;
__global__ void mlp_t_reduce_kernel(const float* tpart, int M_pad, int slots, int n_tiles, int n_blocks, int n_pairs,
                                    float t_scale, __nv_bfloat16* T) {
  const int mp = blockIdx.x / (2 * kBM / kReduceRows);
  const int r = (blockIdx.x % (2 * kBM / kReduceRows)) * kReduceRows + threadIdx.x / kMlpDownRP;
  const int c = threadIdx.x % kMlpDownRP;
  const int m = mp * 2 * kBM + r;
  const int used = mlp_block_pairs(mp, n_blocks, n_tiles, n_pairs);  // pairs whose range holds a tile of this block
  if (m >= M_pad) return;
  const float* src = tpart + (static_cast<size_t>(mp) * slots * (2 * kBM) + r) * kMlpDownRP + c;
  const int n = used < slots ? used : slots;
  // the slots' loads all in flight at once (up to kReduceUnroll), summed in slot order
  float acc = 0.f;
  for (int s0 = 0; s0 < n; s0 += kReduceUnroll) {
    float v[kReduceUnroll];
#pragma unroll
    for (int u = 0; u < kReduceUnroll; ++u)
      v[u] = s0 + u < n ? src[static_cast<size_t>(s0 + u) * (2 * kBM) * kMlpDownRP] : 0.f;
#pragma unroll
    for (int u = 0; u < kReduceUnroll; ++u)
      if (s0 + u < n) acc += v[u];
  }
  T[static_cast<size_t>(m) * kMlpDownRP + c] = __float2bfloat16_rn(acc * t_scale);
}

int max_pairs_on_device() {
  static std::atomic<int> max_pairs_by_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 74;
  }
  int max_pairs = (dev >= 0 && dev < 64) ? max_pairs_by_dev[dev].load() : 0;
  if (max_pairs <= 0) {
    cudaFuncSetAttribute(gemm_nvfp4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SmemNv<false>::kTotal);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SmemNv<false>::kTotal;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm_nvfp4_kernel<false>, &cfg) != cudaSuccess || clusters < 1) {
      cudaGetLastError();
      int sms = 148;
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      clusters = sms / 2;
    }
    max_pairs = clusters;
    if (dev >= 0 && dev < 64) max_pairs_by_dev[dev].store(max_pairs);
  }
  return max_pairs;
}

template <bool kMlp>
cudaError_t launch(const GemmParams& p, const MlpDownParams& mlp, const GemmMaps& maps, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(gemm_nvfp4_kernel<kMlp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmemNv<kMlp>::kTotal);
  });
  if (e != cudaSuccess) return e;
  if (p.N_pad % kBN != 0) return cudaErrorInvalidValue;
  const int tiles = ((p.M_pad + 255) / 256) * (p.N_pad / kBN);
  const int pairs = nvfp4_pairs(tiles);
  gemm_nvfp4_kernel<kMlp><<<2 * pairs, kThreads, SmemNv<kMlp>::kTotal, stream>>>(p, mlp, maps);
  return cudaGetLastError();
}

}  // namespace

int nvfp4_pairs(int tiles) {
  const int max_pairs = max_pairs_on_device();
  return tiles < max_pairs ? tiles : max_pairs;
}

int nvfp4_mlp_slots(int tiles, int n_blocks, int pairs) {
  int slots = 1;
  for (int mp = 0; mp < tiles / n_blocks; ++mp) {
    const int used = mlp_block_pairs(mp, n_blocks, tiles, pairs);
    slots = used > slots ? used : slots;
  }
  return slots;
}

cudaError_t launch_gemm_nvfp4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream) {
  return launch<false>(p, MlpDownParams{}, maps, stream);
}

cudaError_t launch_gemm_nvfp4_mlp(const GemmParams& p, const MlpDownParams& mlp, const GemmMaps& maps,
                                  cudaStream_t stream) {
  if (!mlp.codes || !mlp.scales || !mlp.tpart || !mlp.inv_s || mlp.K != p.N || mlp.M_pad < p.M_pad)
    return cudaErrorInvalidValue;
  return launch<true>(p, mlp, maps, stream);
}

cudaError_t launch_mlp_t_reduce(const float* tpart, int M_pad, int slots, int tiles, int n_blocks, int pairs,
                                float t_scale, __nv_bfloat16* T, cudaStream_t stream) {
  const int m_blocks = (M_pad + 255) / 256;
  mlp_t_reduce_kernel<<<m_blocks * (2 * kBM / kReduceRows), kReduceRows * kMlpDownRP, 0, stream>>>(tpart, M_pad, slots, tiles, n_blocks, pairs, t_scale, T);
  return cudaGetLastError();
}

}  // namespace svdq
