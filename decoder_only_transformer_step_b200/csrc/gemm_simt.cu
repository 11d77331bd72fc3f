// fp32 CUDA-core GEMM for the correctness mode (mode 1): the same products and
// fused epilogues as the tensor-core path, with fp32 FMA accumulation, for
// tight parity checks on small shapes.  Generic strides cover every operand
// majorness; 64 x 64 output tile, 4 x 4 outputs per thread.
#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_simt_kernel(const GemmArgs g) {
  pdl_start();
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const float* A = (const float*)g.A;
  const float* B = (const float*)g.B;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += TK) {
    for (int i = threadIdx.x; i < TK * TM; i += 256) {
      int kk, mm;
      if (g.a_mn) { kk = i / TM; mm = i % TM; } else { mm = i / TK; kk = i % TK; }
      int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < g.M && k < g.K) v = g.a_mn ? A[(long)k * g.lda + m] : A[(long)m * g.lda + k];
      As[kk][mm] = v;
    }
    for (int i = threadIdx.x; i < TK * TN; i += 256) {
      int kk, nn;
      if (g.b_mn) { kk = i / TN; nn = i % TN; } else { nn = i / TK; kk = i % TK; }
      int n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < g.N && k < g.K) v = g.b_mn ? B[(long)k * g.ldb + n] : B[(long)n * g.ldb + k];
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < g.M && n < g.N) epi_one<float>(g.epi, nullptr, 0, g.M, g.N, m, n, acc[i][j]);
    }
}

}  // namespace

int gemm_simt_f32(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return GPT2_OK;
  if (g.epi.kind == EPI_F32_PARTIAL) return GPT2_ERR_INVALID_ARG;
  dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM);
  CUDA_TRY(launch_k(gemm_simt_kernel, grid, 256, 0, st, g));
  LAUNCH_CHECK();
  return GPT2_OK;
}
