// Offline SVDQuant steps on the GPU (msModelSlim SVDQuant entry, section 2.1:
// migrate -> decompose -> quantize the residual; section 2.3 eqs. 1-3).
// These run once per layer; they are simple elementwise / reduction kernels.
// The quantizers reproduce the activation kernel's arithmetic exactly, so the
// weight codes and scales are bit-identical to what the CPU oracle computes.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Round a double to the nearest bfloat16 (ties to even) without going through
// float (no double rounding): a value in [2^(e-1), 2^e) keeps 8 significant
// bits, i.e. its last place is 2^(e-8); below 2^-126 the last place is 2^-133.
__device__ __forceinline__ __nv_bfloat16 bf16_from_double(double x) {
  if (x == 0.0) return __ushort_as_bfloat16(signbit(x) ? 0x8000 : 0);
  int e;
  frexp(x, &e);
  const int ue = max(e - 8, -133);
  const double r = ldexp(rint(ldexp(x, -ue)), ue);
  return __float2bfloat16_rz(static_cast<float>(r));  // exact: r is a bfloat16 value
}

__global__ void absmax_rows_kernel(const __nv_bfloat16* W, int K, int N, float* out) {
  const int k = blockIdx.x;
  float m = 0.f;
  for (int n = threadIdx.x; n < N; n += blockDim.x) m = fmaxf(m, fabsf(__bfloat162float(W[static_cast<size_t>(k) * N + n])));
  m = warp_max(m);
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) out[k] = v;
  }
}

// running_max[k] = max(running_max[k], max_m |X[m,k]|); values are >= 0, so
// the float bit patterns order like unsigned integers.
__global__ void absmax_cols_kernel(const __nv_bfloat16* X, int M, int K, float* running) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const int rows_per = (M + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * rows_per, r1 = min(M, r0 + rows_per);
  float m = 0.f;
  for (int r = r0; r < r1; ++r) m = fmaxf(m, fabsf(__bfloat162float(X[static_cast<size_t>(r) * K + k])));
  atomicMax(reinterpret_cast<unsigned int*>(running) + k, __float_as_uint(m));
}

__global__ void migrate_kernel(const __nv_bfloat16* W, const float* s, int K, int N, float* W_hat) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(K) * N) return;
  const int k = static_cast<int>(i / N);
  W_hat[i] = __fmul_rn(s[k], __bfloat162float(W[i]));
}

// W_hat [K,N] row-major -> float64, column-major. transpose=false keeps the
// memory order (the column-major N x K matrix W_hat^T); true writes the
// column-major K x N matrix W_hat.
__global__ void to_f64_kernel(const float* W_hat, int K, int N, bool transpose, double* out) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(K) * N) return;
  if (!transpose) {
    out[i] = static_cast<double>(W_hat[i]);
  } else {
    const int k = static_cast<int>(i / N), n = static_cast<int>(i % N);
    out[k + static_cast<size_t>(n) * K] = static_cast<double>(W_hat[i]);
  }
}

// One block per rank component j: L1[:,j] = u_j, L2[j,:] = sigma_j v_j^T, the
// sign chosen so that the largest-magnitude entry of u_j is positive, both
// rounded to bfloat16.
//  wt = true : the SVD was of W_hat^T (N x K, N >= K) = U' S V'^T, so
//              u_j[k] = VT[j + k*ldvt], v_j[n] = U[n + j*ldu]
//  wt = false: the SVD was of W_hat (K x N, K > N) = U S V^T, so
//              u_j[k] = U[k + j*ldu],   v_j[n] = VT[j + n*ldvt]
__global__ void factors_kernel(const double* U, const double* S, const double* VT, int K, int N, bool wt, int ldu,
                               int ldvt, __nv_bfloat16* L1, __nv_bfloat16* L2, int rank) {
  const int j = blockIdx.x;
  auto u_at = [&](int k) -> double { return wt ? VT[j + static_cast<size_t>(k) * ldvt] : U[k + static_cast<size_t>(j) * ldu]; };
  auto v_at = [&](int n) -> double { return wt ? U[n + static_cast<size_t>(j) * ldu] : VT[j + static_cast<size_t>(n) * ldvt]; };
  // argmax |u_j| (first index on ties)
  double best = -1.0;
  int bi = 0x7fffffff;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double a = fabs(u_at(k));
    if (a > best || (a == best && k < bi)) { best = a; bi = k; }
  }
  __shared__ double sb[1024];
  __shared__ int si[1024];
  sb[threadIdx.x] = best;
  si[threadIdx.x] = bi;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      const double a = sb[threadIdx.x + o];
      const int i = si[threadIdx.x + o];
      if (a > sb[threadIdx.x] || (a == sb[threadIdx.x] && i < si[threadIdx.x])) {
        sb[threadIdx.x] = a;
        si[threadIdx.x] = i;
      }
    }
    __syncthreads();
  }
  const double sign = u_at(si[0]) < 0.0 ? -1.0 : 1.0;
  const double sigma = S[j];
  for (int k = threadIdx.x; k < K; k += blockDim.x) L1[static_cast<size_t>(k) * rank + j] = bf16_from_double(sign * u_at(k));
  for (int n = threadIdx.x; n < N; n += blockDim.x) L2[static_cast<size_t>(j) * N + n] = bf16_from_double(sign * sigma * v_at(n));
}

// R = fp32(W_hat - sum_j L1[:,j] L2[j,:]) in float64, terms subtracted in the
// order j = 0..rank-1 (each bf16 x bf16 product is exact in float64).
__global__ void residual_kernel(const float* W_hat, const __nv_bfloat16* L1, const __nv_bfloat16* L2, int K, int N,
                                int rank, float* R) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int k = blockIdx.y;
  if (n >= N) return;
  double acc = static_cast<double>(W_hat[static_cast<size_t>(k) * N + n]);
  const __nv_bfloat16* l1 = L1 + static_cast<size_t>(k) * rank;
  for (int j = 0; j < rank; ++j) {
    const double a = static_cast<double>(__bfloat162float(l1[j]));
    const double b = static_cast<double>(__bfloat162float(L2[static_cast<size_t>(j) * N + n]));
    acc = __dsub_rn(acc, __dmul_rn(a, b));
  }
  R[static_cast<size_t>(k) * N + n] = __double2float_rn(acc);
}

__global__ void absmax_all_kernel(const float* v, size_t n, unsigned int* out) {
  float m = 0.f;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += static_cast<size_t>(gridDim.x) * blockDim.x)
    m = fmaxf(m, fabsf(v[i]));
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

// INT4 g64 weight codes: thread per (output column n, group g). Codes are the
// E4M3 bytes of the integers (exact), laid out [N_pad, K]; scales [K/64][N_pad].
__global__ void quant_w_int4_kernel(const float* R, int K, int N, int N_pad, uint8_t* codes8, float* sw) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (n >= N) return;
  float v[64];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    v[i] = R[static_cast<size_t>(g * 64 + i) * N + n];
    amax = fmaxf(amax, fabsf(v[i]));
  }
  float scale = 0.f;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = 0;
  if (amax > 0.f) {
    scale = __fdiv_rn(amax, 7.0f);
    const float inv = __fdiv_rn(7.0f, amax);
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
      const int q0 = min(7, max(-8, __float2int_rn(__fmul_rn(v[i], inv))));
      const int q1 = min(7, max(-8, __float2int_rn(__fmul_rn(v[i + 1], inv))));
      w[i >> 2] |= cvt_e4m3x2(static_cast<float>(q0), static_cast<float>(q1)) << (16 * ((i >> 1) & 1));
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(codes8 + static_cast<size_t>(n) * K + g * 64);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  sw[static_cast<size_t>(g) * N_pad + n] = scale;
}

// NVFP4 weight codes: thread per (n, 16-element block b). The tensor scale
// g_w = amax(R) / 2688 is derived here from the reduced amax bits.
__global__ void quant_w_nvfp4_kernel(const float* R, int K, int N, const unsigned int* amax_bits, uint8_t* codes4,
                                     uint8_t* sf_atoms, float* g_w_out) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  const float amax_t = __uint_as_float(*amax_bits);
  const float g = amax_t == 0.f ? 1.0f : __fdiv_rn(amax_t, 2688.0f);
  if (n == 0 && b == 0) *g_w_out = g;
  if (n >= N) return;
  const float denom = __fmul_rn(6.0f, g);
  float v[16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = R[static_cast<size_t>(b * 16 + i) * N + n];
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const uint32_t sb = cvt_e4m3x2(__fdiv_rn(amax, denom), 0.f) & 0xFFu;
  const float eff = __fmul_rn(e4m3_to_float(sb), g);
  uint32_t c0 = 0, c1 = 0;
  if (eff != 0.f) {
    const float inv = __frcp_rn(eff);
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], inv);
    c0 = cvt_e2m1x8(q);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[8 + i], inv);
    c1 = cvt_e2m1x8(q);
  }
  *reinterpret_cast<uint2*>(codes4 + static_cast<size_t>(n) * (K / 2) + b * 8) = make_uint2(c0, c1);
  const size_t atom = static_cast<size_t>(n >> 7) * (K >> 6) + (b >> 2);
  sf_atoms[atom * 512 + (n & 31) * 16 + ((n >> 5) & 3) * 4 + (b & 3)] = static_cast<uint8_t>(sb);
}

// One block of the low-rank branch (the base factors, or one LoRA adapter)
// written at branch columns [c0, c0 + rb):
//   L1T [RP, K]   <- F^T         (the canonical input-side factor)
//   L1sTh, L1sTl  <- hi / lo of fp32(inv_s[k] * F[k, j]): hi = bf16(v),
//                    lo = bf16(v - hi) (the difference is exact in float), the
//                    factor with 1/s folded in that the activation kernel uses
//   L2T [N_pad, RP] <- G^T       (the output-side factor)
// F is [K, rb] and G is [rb, N], both row-major bf16. Columns outside every
// block stay as the caller zeroed them.
__global__ void assemble_block_kernel(const __nv_bfloat16* F, const __nv_bfloat16* G, int rb, int c0, int K, int N,
                                      int RP, const float* inv_s, __nv_bfloat16* L1T, __nv_bfloat16* L1sTh,
                                      __nv_bfloat16* L1sTl, __nv_bfloat16* L2T) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t n1 = static_cast<size_t>(rb) * K;
  const size_t n2 = static_cast<size_t>(rb) * N;
  if (i < n1) {
    const int j = static_cast<int>(i / K), k = static_cast<int>(i % K);
    const __nv_bfloat16 f = F[static_cast<size_t>(k) * rb + j];
    const size_t o = static_cast<size_t>(c0 + j) * K + k;
    L1T[o] = f;
    const float v = __fmul_rn(inv_s[k], __bfloat162float(f));
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    L1sTh[o] = hi;
    L1sTl[o] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
  } else if (i < n1 + n2) {
    const size_t t = i - n1;
    const int j = static_cast<int>(t / N), n = static_cast<int>(t % N);
    L2T[static_cast<size_t>(n) * RP + c0 + j] = G[t];
  }
}

// The factors of a LoRA adapter as the branch sees them. The branch input is
// x_hat = X diag(s)^-1, so X A = x_hat (diag(s) A): F = bf16(s[k] * A[k, j])
// [K, r_l] and G = bf16(scale * B[j, n]) [r_l, N]; each product is exact in
// float64 and rounded once.
__global__ void lora_factors_kernel(const __nv_bfloat16* A, const __nv_bfloat16* B, int K, int N, int r_l, float scale,
                                    const float* s, __nv_bfloat16* F, __nv_bfloat16* G) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t n1 = static_cast<size_t>(K) * r_l;
  const size_t n2 = static_cast<size_t>(r_l) * N;
  if (i < n1) {
    const int k = static_cast<int>(i / r_l);
    F[i] = bf16_from_double(static_cast<double>(s[k]) * static_cast<double>(__bfloat162float(A[i])));
  } else if (i < n1 + n2) {
    const size_t t = i - n1;
    G[t] = bf16_from_double(static_cast<double>(scale) * static_cast<double>(__bfloat162float(B[t])));
  }
}

// Failure-detection self-test: waits on an mbarrier that nothing ever
// arrives on, with the same bounded wait the GEMM pipelines use, and reports
// the outcome through the status word.
__global__ void wait_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t a = smem_u32(&bar);
    const uint64_t t0 = globaltimer_ns();
    bool done = false;
    while (!done) {
      done = mbar_try_wait(a, 0);
      if (!done && globaltimer_ns() - t0 > limit_ns) {
        atomicExch(status, kDevTimeout);
        break;
      }
    }
    if (done) atomicExch(status, kDevOk);
  }
}

inline unsigned blocks_for(size_t n, int t) { return static_cast<unsigned>((n + t - 1) / t); }

}  // namespace

cudaError_t launch_absmax_rows(const __nv_bfloat16* W, int K, int N, float* out, cudaStream_t s) {
  absmax_rows_kernel<<<K, 256, 0, s>>>(W, K, N, out);
  return cudaGetLastError();
}
cudaError_t launch_absmax_cols(const __nv_bfloat16* X, int M, int K, float* running, cudaStream_t s) {
  dim3 grid((K + 255) / 256, max(1, min(64, M / 64)));
  absmax_cols_kernel<<<grid, 256, 0, s>>>(X, M, K, running);
  return cudaGetLastError();
}
cudaError_t launch_migrate(const __nv_bfloat16* W, const float* s_k, int K, int N, float* W_hat, cudaStream_t st) {
  migrate_kernel<<<blocks_for(static_cast<size_t>(K) * N, 256), 256, 0, st>>>(W, s_k, K, N, W_hat);
  return cudaGetLastError();
}
cudaError_t launch_to_f64_colmajor(const float* W_hat, int K, int N, bool transpose, double* out, cudaStream_t st) {
  to_f64_kernel<<<blocks_for(static_cast<size_t>(K) * N, 256), 256, 0, st>>>(W_hat, K, N, transpose, out);
  return cudaGetLastError();
}
cudaError_t launch_factors_from_svd(const double* U, const double* S, const double* VT, int K, int N, int rank, bool wt,
                                    int ldu, int ldvt, __nv_bfloat16* L1, __nv_bfloat16* L2, cudaStream_t st) {
  factors_kernel<<<rank, 1024, 0, st>>>(U, S, VT, K, N, wt, ldu, ldvt, L1, L2, rank);
  return cudaGetLastError();
}
cudaError_t launch_residual(const float* W_hat, const __nv_bfloat16* L1, const __nv_bfloat16* L2, int K, int N, int rank,
                            float* R, cudaStream_t st) {
  dim3 grid((N + 255) / 256, K);
  residual_kernel<<<grid, 256, 0, st>>>(W_hat, L1, L2, K, N, rank, R);
  return cudaGetLastError();
}
cudaError_t launch_absmax_all(const float* R, size_t n, unsigned int* out_bits, cudaStream_t st) {
  absmax_all_kernel<<<1184, 256, 0, st>>>(R, n, out_bits);
  return cudaGetLastError();
}
cudaError_t launch_quant_weight_int4(const float* R, int K, int N, int N_pad, uint8_t* codes8, float* sw,
                                     cudaStream_t st) {
  dim3 grid((N + 127) / 128, K / 64);
  quant_w_int4_kernel<<<grid, 128, 0, st>>>(R, K, N, N_pad, codes8, sw);
  return cudaGetLastError();
}
cudaError_t launch_quant_weight_nvfp4(const float* R, int K, int N, int N_pad, const unsigned int* amax_bits,
                                      uint8_t* codes4, uint8_t* sf_atoms, float* g_w_out, cudaStream_t st) {
  (void)N_pad;
  dim3 grid((N + 127) / 128, K / 16);
  quant_w_nvfp4_kernel<<<grid, 128, 0, st>>>(R, K, N, amax_bits, codes4, sf_atoms, g_w_out);
  return cudaGetLastError();
}
cudaError_t launch_assemble_block(const __nv_bfloat16* F, const __nv_bfloat16* G, int rb, int c0, int K, int N,
                                  int RP, const float* inv_s, __nv_bfloat16* L1T, __nv_bfloat16* L1sTh,
                                  __nv_bfloat16* L1sTl, __nv_bfloat16* L2T, cudaStream_t st) {
  const size_t n = static_cast<size_t>(rb) * (K + N);
  if (n == 0) return cudaSuccess;
  assemble_block_kernel<<<blocks_for(n, 256), 256, 0, st>>>(F, G, rb, c0, K, N, RP, inv_s, L1T, L1sTh, L1sTl, L2T);
  return cudaGetLastError();
}
cudaError_t launch_lora_factors(const __nv_bfloat16* A, const __nv_bfloat16* B, int K, int N, int r_l, float scale,
                                const float* s_k, __nv_bfloat16* F, __nv_bfloat16* G, cudaStream_t st) {
  const size_t n = static_cast<size_t>(r_l) * (K + N);
  lora_factors_kernel<<<blocks_for(n, 256), 256, 0, st>>>(A, B, K, N, r_l, scale, s_k, F, G);
  return cudaGetLastError();
}
cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace svdq
