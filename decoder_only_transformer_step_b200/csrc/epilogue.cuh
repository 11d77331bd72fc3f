// GEMM epilogue of one element for the CUDA-core GEMM of the fp32 mode: the
// bias, residual, GELU and GELU' steps of a decoder block fused into the store
// of the matmul result, plus the fp32 weight-gradient store (beta * old +
// alpha * acc).  The tensor-core GEMM has its own vectorised form of the same
// arithmetic.
#pragma once

#include "common.cuh"
#include "internal.h"

template <typename T>
DEVI void epi_one(const EpiArgs& e, float* partial, int split, int M, int N, int row, int col,
                  float v) {
  constexpr bool FAST = sizeof(T) == 2;
  const long idx = (long)row * e.ldo + col;
  switch (e.kind) {
    case EPI_STORE:
    case EPI_ROWDOT:  // (the row sums need the tensor-core epilogue; here only the store)
      ((T*)e.out)[idx] = from_f<T>(e.alpha * v);
      break;
    case EPI_BIAS:
      ((T*)e.out)[idx] = from_f<T>(v + to_f(((const T*)e.bias)[col]));
      break;
    case EPI_BIAS_RESID:
      ((T*)e.out)[idx] =
          from_f<T>(v + to_f(((const T*)e.bias)[col]) + to_f(((const T*)e.resid)[idx]));
      break;
    case EPI_BIAS_GELU: {
      float gl, dg;
      gelu_and_grad_f<FAST>(v + to_f(((const T*)e.bias)[col]), gl, dg);
      ((T*)e.out)[idx] = from_f<T>(dg);
      ((T*)e.out2)[idx] = from_f<T>(gl);
      break;
    }
    case EPI_DGELU:
      ((T*)e.out)[idx] = from_f<T>(v * to_f(((const T*)e.aux)[idx]));
      break;
    case EPI_F32: {
      float* o = (float*)e.out;
      o[idx] = (e.beta != 0.f ? e.beta * o[idx] : 0.f) + e.alpha * v;
      break;
    }
    case EPI_F32_PARTIAL:
      partial[((long)split * M + row) * N + col] = v;
      break;
  }
}
