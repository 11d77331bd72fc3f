// GEMM epilogues: the bias, residual, GELU and GELU' steps of a decoder block
// fused into the store of the matmul result, plus the fp32 weight-gradient
// store (beta * old + alpha * acc).
#pragma once

#include "common.cuh"
#include "internal.h"

// One element (used by the CUDA-core GEMM and by ragged tile edges).
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

// ---- 32 consecutive bf16 columns of one row, 16-byte vector accesses ----

DEVI void ld_bf16x32(const bf16* p, float (&f)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u = q[i];
    f[8 * i + 0] = bf16lo(u.x); f[8 * i + 1] = bf16hi(u.x);
    f[8 * i + 2] = bf16lo(u.y); f[8 * i + 3] = bf16hi(u.y);
    f[8 * i + 4] = bf16lo(u.z); f[8 * i + 5] = bf16hi(u.z);
    f[8 * i + 6] = bf16lo(u.w); f[8 * i + 7] = bf16hi(u.w);
  }
}
DEVI void st_bf16x32(bf16* p, const float (&f)[32]) {
  uint4* q = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16x2(f[8 * i + 0], f[8 * i + 1]);
    u.y = pack_bf16x2(f[8 * i + 2], f[8 * i + 3]);
    u.z = pack_bf16x2(f[8 * i + 4], f[8 * i + 5]);
    u.w = pack_bf16x2(f[8 * i + 6], f[8 * i + 7]);
    q[i] = u;
  }
}

DEVI void unpack8(const uint4& u, float* f) {
  f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
  f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}

// Epilogue arithmetic for 32 accumulators of one row, without the store (the
// tensor-core path stages the result in shared memory and stores it with TMA,
// which clips rows >= M and columns >= N).  `op` holds the residual
// (EPI_BIAS_RESID) or saved GELU'(u) (EPI_DGELU) chunk, read from its TMA box.  For EPI_BIAS_GELU
// v becomes u = acc + bias; the caller derives GELU(u) and GELU'(u) from it.
DEVI void epi_apply_row32(const EpiArgs& e, int N, int col0, float (&v)[32], const uint4 (&op)[4]) {
  const bool need_bias = e.kind == EPI_BIAS || e.kind == EPI_BIAS_RESID || e.kind == EPI_BIAS_GELU;
  if (need_bias) {
    const bf16* b = (const bf16*)e.bias + col0;
    if (col0 + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float t[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(b) + i), t);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * i + j] += t[j];
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < N) v[j] += to_f(b[j]);
    }
  }
  if (e.kind == EPI_BIAS_RESID) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t[8];
      unpack8(op[i], t);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * i + j] += t[j];
    }
  } else if (e.kind == EPI_DGELU) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float t[8];
      unpack8(op[i], t);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * i + j] *= t[j];
    }
  } else if (e.kind == EPI_STORE || e.kind == EPI_F32 || e.kind == EPI_ROWDOT) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= e.alpha;
  }
}

// Row `lane` of a 32 x 32 staging box: bf16 rows of 64 B in the TMA 64-byte
// swizzle (16-byte chunk j of row r at chunk j ^ ((r >> 1) & 3)); fp32 rows of
// 128 B in the 128-byte swizzle (chunk j ^ (r & 7)).  Both keep a warp's
// 16-byte stores spread over all 32 banks.
DEVI void stage_bf16_row(uint32_t box, int lane, const float (&v)[32]) {
  const uint32_t rb = box + (uint32_t)lane * 64u;
  const int x = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_shared_v4(rb + 16u * (uint32_t)(j ^ x), pack_bf16x2(v[8 * j], v[8 * j + 1]),
                 pack_bf16x2(v[8 * j + 2], v[8 * j + 3]), pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                 pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}
// Row `lane` of a bf16 32 x 32 box in the 64-byte swizzle (as TMA loads it),
// as four 16-byte words in column order.
DEVI void load_bf16_box_row(uint32_t box, int lane, uint4 (&u)[4]) {
  const uint32_t rb = box + (uint32_t)lane * 64u;
  const int x = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(u[j].x), "=r"(u[j].y), "=r"(u[j].z), "=r"(u[j].w)
                 : "r"(rb + 16u * (uint32_t)(j ^ x)));
}
// GELU'(u) into `box` and GELU(u) into `box2` (the stage_bf16_row layout),
// eight columns at a time from one tanh each.
DEVI void stage_gelu_pair_row(uint32_t box, uint32_t box2, int lane, const float (&u)[32]) {
  const uint32_t rb = box + (uint32_t)lane * 64u, rb2 = box2 + (uint32_t)lane * 64u;
  const int x = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float g[8], dg[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) gelu_and_grad_f<true>(u[8 * j + i], g[i], dg[i]);
    const uint32_t off = 16u * (uint32_t)(j ^ x);
    st_shared_v4(rb + off, pack_bf16x2(dg[0], dg[1]), pack_bf16x2(dg[2], dg[3]), pack_bf16x2(dg[4], dg[5]),
                 pack_bf16x2(dg[6], dg[7]));
    st_shared_v4(rb2 + off, pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]), pack_bf16x2(g[4], g[5]),
                 pack_bf16x2(g[6], g[7]));
  }
}

DEVI void stage_f32_row(uint32_t box, int lane, const float (&v)[32]) {
  const uint32_t rb = box + (uint32_t)lane * 128u;
  const int x = lane & 7;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_shared_v4(rb + 16u * (uint32_t)(j ^ x), __float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                 __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
}

// Full chunk: row < M and col0 + 32 <= N, all row pitches multiples of 8.
DEVI void epi_row32_bf16(const EpiArgs& e, float* partial, int split, int M, int N, int row,
                         int col0, float (&v)[32]) {
  const long idx = (long)row * e.ldo + col0;
  float t[32];
  switch (e.kind) {
    case EPI_STORE:
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= e.alpha;
      st_bf16x32((bf16*)e.out + idx, v);
      break;
    case EPI_BIAS:
      ld_bf16x32((const bf16*)e.bias + col0, t);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += t[j];
      st_bf16x32((bf16*)e.out + idx, v);
      break;
    case EPI_BIAS_RESID:
      ld_bf16x32((const bf16*)e.bias + col0, t);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += t[j];
      ld_bf16x32((const bf16*)e.resid + idx, t);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += t[j];
      st_bf16x32((bf16*)e.out + idx, v);
      break;
    case EPI_BIAS_GELU:
      ld_bf16x32((const bf16*)e.bias + col0, t);
#pragma unroll
      for (int j = 0; j < 32; ++j) gelu_and_grad_f<true>(v[j] + t[j], t[j], v[j]);
      st_bf16x32((bf16*)e.out + idx, v);   // GELU'(u)
      st_bf16x32((bf16*)e.out2 + idx, t);  // GELU(u)
      break;
    case EPI_DGELU:
      ld_bf16x32((const bf16*)e.aux + idx, t);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= t[j];
      st_bf16x32((bf16*)e.out + idx, v);
      break;
    case EPI_F32: {
      float4* o = reinterpret_cast<float4*>((float*)e.out + idx);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e.beta != 0.f) {
          r = o[i];
          r.x *= e.beta; r.y *= e.beta; r.z *= e.beta; r.w *= e.beta;
        }
        r.x += e.alpha * v[4 * i + 0];
        r.y += e.alpha * v[4 * i + 1];
        r.z += e.alpha * v[4 * i + 2];
        r.w += e.alpha * v[4 * i + 3];
        o[i] = r;
      }
      break;
    }
    case EPI_F32_PARTIAL: {
      float4* o = reinterpret_cast<float4*>(partial + ((long)split * M + row) * N + col0);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      break;
    }
  }
}
