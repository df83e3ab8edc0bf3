// Internal launch interfaces of the SVDQuant kernels (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace svdq {

// A 2-D tiled TMA map over a row-major [outer, inner] tensor (row_bytes
// between rows), box {box_inner, box_outer}; false if encoding failed.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);

// LoRA adapter slots a layer can hold at once (bit s of a row's adapter mask
// selects slot s).
constexpr int kMaxAdapters = 8;

// ---------------------------------------------------------------- K1
struct ActQuantParams {
  const __nv_bfloat16* X;  // [M, K] row-major
  int M, K, M_pad;         // M_pad = roundup(M, 128)
  const float* inv_s;      // [K]
  uint8_t* codes;          // INT4: [M_pad, K] E4M3 bytes of the integer codes; NVFP4: [M_pad, K/2] packed E2M1
  void* scales;            // INT4: float [K/64][M_pad]; NVFP4: scale-factor atoms [M_pad/128][K/64][512]
  __nv_bfloat16* T;        // [M_pad, RP] bf16 = t_scale * (x_hat L1)
  __nv_bfloat16* T_lo;     // NULL, or [M_pad, RP]: bf16(v - T) of the same float v (T + T_lo ~ 16 bits of v)
  int split;               // K shares per 128-row block (from act_quant_split)
  float* Tpart;            // [split][M_pad][RP] float partials over the K shares (split > 1)
  int* counters;           // [M_pad / 128] arrival counts of the shares, zero between launches
  float g_x;               // NVFP4 activation tensor scale
  float denom;             // NVFP4: fp32(6 * g_x)
  float t_scale;           // 1 (INT4) or 1 / (g_x g_w) (NVFP4)
  int* status;             // device status word (kDevTimeout on a given-up wait)
  // Per-row LoRA adapter selection: bit s of row_mask[m] keeps the T columns
  // of adapter slot s for row m ([col_start[s], col_start[s+1])); the base
  // factor's columns [0, col_start[0]) are always kept. NULL keeps everything.
  const uint32_t* row_mask;  // [M] or NULL
  int col_start[kMaxAdapters + 1];
};
struct ActQuantMaps {
  CUtensorMap x;    // X [M, K] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap l1h;  // L1s^T high part [RP, K] bf16, box {64, RP}, 128-byte swizzle
  CUtensorMap l1l;  // L1s^T low part  [RP, K] bf16, box {64, RP}, 128-byte swizzle
};
int act_quant_box_rows();
// Resident activation-kernel CTAs per SM for (format, rank padding) on the
// current device (an occupancy query; call it once per layer, not per launch).
int act_quant_resident(int fmt, int rp);
// K shares per 128-row block for M_pad rows, so that the grid fills the GPU in
// one wave: a pure function of its arguments.
int act_quant_split(int M_pad, int K, int per_sm, int sms);
// Row blocks the per-layer arrival counters cover (M_pad / 128 at most this).
constexpr int kMaxRowBlocks = 65536;
cudaError_t launch_act_quant(const ActQuantParams& p, const ActQuantMaps& maps, int fmt, int rp, cudaStream_t stream);

// ---------------------------------------------------------------- GEMMs
struct GemmParams {
  int M, N, K, RP;
  __nv_bfloat16* Y;            // [M, N]
  const __nv_bfloat16* bias;   // [N_pad], zero beyond N
  const void* sa;              // activation scales (layout of ActQuantParams::scales)
  const void* sb;              // weight scales: INT4 float [K/64][N_pad]; NVFP4 atoms [N_pad/128][K/64][512]
  int M_pad, N_pad;
  float out_scale;             // NVFP4: g_x g_w; INT4: 1
  int* status;                 // device status word (kDevTimeout on a given-up wait)
};
struct GemmMaps {
  CUtensorMap a;    // activation codes
  CUtensorMap b;    // weight codes
  CUtensorMap t;    // T [M_pad, RP] bf16
  CUtensorMap l2;   // L2T [N_pad, RP] bf16
  CUtensorMap sfa;  // NVFP4 activation scale-factor atoms as uint32 [atoms, 128], box {128, 4}
  CUtensorMap sfb;  // NVFP4 weight scale-factor atoms, same view
  CUtensorMap y;    // NVFP4: Y [M, N] bf16, box {32, 32}, 64-byte swizzle (TMA stores)
  CUtensorMap l1h_down;  // MLP block: the down layer's L1s^T high part [RP_down, K_down], box {64, RP_down / 2}
  CUtensorMap l1l_down;  // ... and low part
  CUtensorMap t_lo;      // MLP block: the up layer's T low part [M_pad, RP] bf16, as t
};

// The down layer of an MLP block as the fused epilogue of the up layer's
// NVFP4 GEMM sees it: GELU of the up output is smoothed and quantized
// straight into the down layer's activation buffers, and its branch input T
// is accumulated from the same tile (partials over the pairs of SMs, summed
// by mlp_t_reduce_kernel).
constexpr int kMlpDownRP = 32;  // branch width of the down layer the fused epilogue supports
struct MlpDownParams {
  int K;                 // the down layer's K (= the up layer's N)
  int M_pad;             // rows of the down layer's activation buffers
  const float* inv_s;    // [K]
  uint8_t* codes;        // [M_pad, K/2] packed E2M1
  uint8_t* scales;       // scale-factor atoms [M_pad/128][K/64][512]
  float g_x, denom;      // the down layer's static activation tensor scale and fp32(6 g_x)
  float* tpart;          // T partials [ceil(M_pad / 256)][slots][256][kMlpDownRP] float
  int slots;             // partial slots per 256-row block
};
// Pairs of SMs the NVFP4 GEMM runs on for `tiles` 256 x 256 tiles (current device).
int nvfp4_pairs(int tiles);
// Partial slots per 256-row block the fused MLP epilogue needs with `pairs` pairs.
int nvfp4_mlp_slots(int tiles, int n_blocks, int pairs);
cudaError_t launch_gemm_nvfp4_mlp(const GemmParams& p, const MlpDownParams& mlp, const GemmMaps& maps,
                                  cudaStream_t stream);
// T = bf16(t_scale * sum of the partials in slot order) [M_pad, kMlpDownRP].
cudaError_t launch_mlp_t_reduce(const float* tpart, int M_pad, int slots, int tiles, int n_blocks, int pairs,
                                float t_scale, __nv_bfloat16* T, cudaStream_t stream);
// Rows of one TMA box of the weight codes, of L2^T and of the activation codes.
// The GEMMs load a tile's operand rows as several boxes: copies in flight,
// not their size, set the TMA throughput of an SM.
constexpr int kWeightBoxRows = 128;
#ifndef SVDQ_ACT_BOX_ROWS
#define SVDQ_ACT_BOX_ROWS 128
#endif
constexpr int kActBoxRows = SVDQ_ACT_BOX_ROWS;
cudaError_t launch_gemm_nvfp4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream);
cudaError_t launch_gemm_int4(const GemmParams& p, const GemmMaps& maps, cudaStream_t stream);

// ---------------------------------------------------------------- prepare
cudaError_t launch_absmax_rows(const __nv_bfloat16* W, int K, int N, float* out, cudaStream_t s);
cudaError_t launch_absmax_cols(const __nv_bfloat16* X, int M, int K, float* running_max, cudaStream_t s);
cudaError_t launch_migrate(const __nv_bfloat16* W, const float* s_k, int K, int N, float* W_hat, cudaStream_t st);
cudaError_t launch_to_f64_colmajor(const float* W_hat, int K, int N, bool transpose, double* out, cudaStream_t st);
cudaError_t launch_factors_from_svd(const double* U, const double* S, const double* VT, int K, int N, int rank,
                                    bool wt, int ldu, int ldvt, __nv_bfloat16* L1, __nv_bfloat16* L2,
                                    cudaStream_t st);
cudaError_t launch_residual(const float* W_hat, const __nv_bfloat16* L1, const __nv_bfloat16* L2, int K, int N,
                            int rank, float* R, cudaStream_t st);
cudaError_t launch_absmax_all(const float* R, size_t n, unsigned int* out_bits, cudaStream_t st);
cudaError_t launch_quant_weight_int4(const float* R, int K, int N, int N_pad, uint8_t* codes8, float* sw,
                                     cudaStream_t st);
cudaError_t launch_quant_weight_nvfp4(const float* R, int K, int N, int N_pad, const unsigned int* amax_bits,
                                      uint8_t* codes4, uint8_t* sf_atoms, float* g_w_out, cudaStream_t st);
// Writes one block of branch columns [c0, c0 + rb) (see prepare_kernels.cu).
cudaError_t launch_assemble_block(const __nv_bfloat16* F, const __nv_bfloat16* G, int rb, int c0, int K, int N,
                                  int RP, const float* inv_s, __nv_bfloat16* L1T, __nv_bfloat16* L1sTh,
                                  __nv_bfloat16* L1sTl, __nv_bfloat16* L2T, cudaStream_t st);
cudaError_t launch_lora_factors(const __nv_bfloat16* A, const __nv_bfloat16* B, int K, int N, int r_l, float scale,
                                const float* s_k, __nv_bfloat16* F, __nv_bfloat16* G, cudaStream_t st);
cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t st);

}  // namespace svdq
