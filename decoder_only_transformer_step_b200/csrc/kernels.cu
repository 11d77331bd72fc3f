// Bandwidth-bound kernels of the GPT-2 step: token + position embedding and
// its (tied, deterministic) backward scatter, LayerNorm forward/backward,
// bias-gradient column sums, the cross-entropy over the padded vocabulary,
// the loss mean, AdamW, and the initialisation.
//
// All accesses are 16-byte vectors along the feature dimension; row
// reductions use warp shuffles; every cross-row reduction is a fixed-order
// two-level sum (per-block partials, then a column reduction), so repeated
// runs give bitwise-identical results.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace {

template <typename T>
struct Vec;  // one 16-byte chunk
template <>
struct Vec<bf16> {
  static constexpr int N = 8;
  DEVI static void load(const bf16* p, float (&f)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
  }
  DEVI static void store(bf16* p, const float (&f)[8]) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  DEVI static void load(const float* p, float (&f)[4]) {
    float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  }
  DEVI static void store(float* p, const float (&f)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

// One 16-byte word as VN floats (the register form of Vec<T>::load).
template <typename T>
DEVI void unpack16(const uint4& u, float (&f)[Vec<T>::N]);
template <>
DEVI void unpack16<bf16>(const uint4& u, float (&f)[8]) {
  f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
  f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}
template <>
DEVI void unpack16<float>(const uint4& u, float (&f)[4]) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y); f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}

// ------------------------------------------------------------- embedding --

// x[m] = wte[tok[m]] + wpe[m mod T]; one warp per row.
template <typename T>
__global__ void embed_fwd_kernel(const int32_t* tok, const T* wte,
                                 const T* wpe, T* __restrict__ x, int M, int Tn, int d,
                                 int vocab_real, int* err) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  const int m = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  int id = tok[m];
  if (id < 0 || id >= vocab_real) {
    if (lane == 0) atomicOr(err, DEV_ERR_TOKEN);
    id = 0;
  }
  const T* a = wte + (long)id * d;
  const T* p = wpe + (long)(m % Tn) * d;
  T* o = x + (long)m * d;
  for (int c = lane * VN; c < d; c += 32 * VN) {
    float fa[VN], fb[VN];
    Vec<T>::load(a + c, fa);
    Vec<T>::load(p + c, fb);
#pragma unroll
    for (int j = 0; j < VN; ++j) fa[j] += fb[j];
    Vec<T>::store(o + c, fa);
  }
}

// Deterministic scatter-add of dx rows into the tied wte gradient: each value
// is rounded once to a 2^-32 fixed-point integer and added with 64-bit
// integer atomics, which are order-independent; then the touched rows are
// converted back and added to dwte (and the accumulator is re-zeroed).
#define FIX_SCALE 4294967296.0

// The fixed point is relative to the backward's grad_scale (fix = 2^32 /
// |grad_scale|): dx is proportional to grad_scale, so the resolution relative
// to the gradient does not shrink under k-fold accumulation (grad_scale 1/k).
template <typename T>
__global__ void embed_scatter_kernel(const int32_t* tok, const T* dx,
                                     unsigned long long* __restrict__ acc, uint8_t* __restrict__ touched,
                                     int M, int d, int V, double fix) {
  pdl_start();
  long i = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (i >= (long)M * d) return;
  const int m = (int)(i / d), c = (int)(i % d);
  int id = tok[m];
  if (id < 0 || id >= V) id = 0;
  double v = (double)to_f(dx[i]) * fix;
  v = fmin(fmax(v, -9.2e18), 9.2e18);
  atomicAdd(acc + (long)id * d + c, (unsigned long long)__double2ll_rn(v));
  if (c == 0) touched[id] = 1;
}

__global__ void embed_convert_kernel(unsigned long long* __restrict__ acc, uint8_t* __restrict__ touched,
                                     float* __restrict__ dwte, int V, int d, double inv_fix) {
  pdl_start();
  const int v = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (v >= V || !touched[v]) return;
  unsigned long long* a = acc + (long)v * d;
  float* g = dwte + (long)v * d;
  for (int c = lane; c < d; c += 32) {
    long long q = (long long)a[c];
    g[c] += (float)((double)q * inv_fix);
    a[c] = 0ull;
  }
  __syncwarp();
  if (lane == 0) touched[v] = 0;
}

// dwpe[t] = (accumulate ? dwpe[t] : 0) + sum_b dx[b, t]   (fixed order in b)
template <typename T>
__global__ void wpe_grad_kernel(const T* dx, float* __restrict__ dwpe, int B, int Tn, int d,
                                int accumulate) {
  pdl_start();
  long i = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (i >= (long)Tn * d) return;
  float s = 0.f;
  for (int b = 0; b < B; ++b) s += to_f(dx[(long)b * Tn * d + i]);
  dwpe[i] = (accumulate ? dwpe[i] : 0.f) + s;
}

// The same with one 16-byte chunk of dx per thread and four batch rows'
// loads in flight (the sum still runs over b in order); for T d a multiple of
// the chunk and 16-byte aligned dx and dwpe.
template <typename T>
__global__ void wpe_grad_vec_kernel(const T* dx, float* __restrict__ dwpe, int B, long tn, int accumulate) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  const long i = (blockIdx.x * (long)blockDim.x + threadIdx.x) * VN;
  if (i >= tn) return;
  float s[VN];
#pragma unroll
  for (int j = 0; j < VN; ++j) s[j] = 0.f;
#pragma unroll 4
  for (int b = 0; b < B; ++b) {
    float f[VN];
    Vec<T>::load(dx + (long)b * tn + i, f);
#pragma unroll
    for (int j = 0; j < VN; ++j) s[j] += f[j];
  }
#pragma unroll
  for (int j = 0; j < VN; j += 4) {
    float4* o = reinterpret_cast<float4*>(dwpe + i + j);
    const float4 old = accumulate ? *o : make_float4(0.f, 0.f, 0.f, 0.f);
    *o = make_float4((accumulate ? old.x : 0.f) + s[j], (accumulate ? old.y : 0.f) + s[j + 1],
                     (accumulate ? old.z : 0.f) + s[j + 2], (accumulate ? old.w : 0.f) + s[j + 3]);
  }
}

// ------------------------------------------------------------- LayerNorm --
// y = (x - mean) * rstd * g + b, mean/var over the row, var biased, eps 1e-5.
// One warp per row; NC = 16-byte chunks per lane (row cached in registers).

template <typename T, int NC>
__global__ void ln_fwd_kernel(const T* x, const T* g, const T* b,
                              T* __restrict__ y, float* __restrict__ mean, float* __restrict__ rstd, int M,
                              int d) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  const int m = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const T* xr = x + (long)m * d;
  float v[NC][VN];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * VN;
    if (c < d) {
      Vec<T>::load(xr + c, v[k]);
#pragma unroll
      for (int j = 0; j < VN; ++j) s += v[k][j];
    }
  }
  const float mu = warp_sum(s) / d;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * VN;
    if (c < d) {
#pragma unroll
      for (int j = 0; j < VN; ++j) {
        float t = v[k][j] - mu;
        q += t * t;
      }
    }
  }
  const float rs = rsqrtf(warp_sum(q) / d + 1e-5f);
  T* yr = y + (long)m * d;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * VN;
    if (c < d) {
      float gg[VN], bb[VN], o[VN];
      Vec<T>::load(g + c, gg);
      Vec<T>::load(b + c, bb);
#pragma unroll
      for (int j = 0; j < VN; ++j) o[j] = (v[k][j] - mu) * rs * gg[j] + bb[j];
      Vec<T>::store(yr + c, o);
    }
  }
  if (lane == 0) {
    mean[m] = mu;
    rstd[m] = rs;
  }
}

// the two bf16 of a packed word as an fp32 pair (low half first)
DEVI float2 bf2w(uint32_t w) { return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); }

// dx = rstd * (dxhat - mean(dxhat) - xhat * mean(dxhat * xhat)), dxhat = dy * g;
// dres = (init ? 0 : dres) + dx.  One warp per row with the row in registers;
// no per-thread accumulators, so many warps are resident to cover HBM latency.
template <typename T, int NC>
__global__ void __launch_bounds__(256) ln_bwd_dx_kernel(const T* dy, const T* x,
                                                        const float* mean,
                                                        const float* rstd,
                                                        const T* g, T* __restrict__ dres,
                                                        int dres_init, int M, int d) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  const int m = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const float mu = mean[m], rs = rstd[m];
  float xh[NC][VN], gd[NC][VN];
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * VN;
    if (c < d) {
      float xv[VN], dv[VN], gv[VN];
      Vec<T>::load(x + (long)m * d + c, xv);
      Vec<T>::load(dy + (long)m * d + c, dv);
      Vec<T>::load(g + c, gv);
#pragma unroll
      for (int j = 0; j < VN; ++j) {
        xh[k][j] = (xv[j] - mu) * rs;
        gd[k][j] = dv[j] * gv[j];
        s1 += gd[k][j];
        s2 += gd[k][j] * xh[k][j];
      }
    }
  }
  s1 = warp_sum(s1) / d;
  s2 = warp_sum(s2) / d;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * VN;
    if (c < d) {
      float o[VN];
      if (!dres_init) {
        Vec<T>::load(dres + (long)m * d + c, o);
      } else {
#pragma unroll
        for (int j = 0; j < VN; ++j) o[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < VN; ++j) o[j] += rs * (gd[k][j] - s1 - xh[k][j] * s2);
      Vec<T>::store(dres + (long)m * d + c, o);
    }
  }
}

// LayerNorm parameter gradients: dgamma = sum_m dy * xhat, dbeta = sum_m dy,
// per block of LNP_ROWS rows (fixed order) into part[rowblock][0:d | d:2d].
constexpr int LNP_ROWS = 128;

template <typename T>
__global__ void __launch_bounds__(256) ln_param_colsum_kernel(const T* dy, const T* x,
                                                              const float* mean,
                                                              const float* rstd, int M, int d,
                                                              float* __restrict__ part) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  __shared__ float red[8][2][32 * VN];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = (blockIdx.x * 32 + lane) * VN;
  const int r0 = blockIdx.y * LNP_ROWS;
  float sg[VN], sb[VN];
#pragma unroll
  for (int j = 0; j < VN; ++j) sg[j] = sb[j] = 0.f;
  if (c < d) {
    for (int r = r0 + warp; r < min(r0 + LNP_ROWS, M); r += 8) {
      const float mu = mean[r], rs = rstd[r];
      float xv[VN], dv[VN];
      Vec<T>::load(x + (long)r * d + c, xv);
      Vec<T>::load(dy + (long)r * d + c, dv);
#pragma unroll
      for (int j = 0; j < VN; ++j) {
        sg[j] += dv[j] * (xv[j] - mu) * rs;
        sb[j] += dv[j];
      }
    }
  }
#pragma unroll
  for (int j = 0; j < VN; ++j) {
    red[warp][0][lane * VN + j] = sg[j];
    red[warp][1][lane * VN + j] = sb[j];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * 32 * VN; i += 256) {
    const int which = i / (32 * VN), k = i % (32 * VN);
    const int col = blockIdx.x * 32 * VN + k;
    if (col < d) {
      float t = red[0][which][k];
      for (int w = 1; w < 8; ++w) t += red[w][which][k];
      part[(long)blockIdx.y * 2 * d + which * d + col] = t;
    }
  }
}

// LayerNorm backward in one pass over dy and x: per row (one warp, the row in
// registers) dres = (init ? 0 : dres) + dx as in ln_bwd_dx_kernel, and per
// lane column accumulators of dgamma = sum dy * xhat, dbeta = sum dy and (for
// RES) sum of the new dres, which is the bias gradient of the linear layer
// that produced this residual-stream gradient.  Rows are dealt to the
// grid's warps round-robin; each block writes its column sums (fixed warp
// order) to part_ln[block][0:d | d:2d] and part_res[block][0:d].
constexpr int LNF_WARPS = 4;
constexpr int LNF_BLOCKS_PER_SM = 3;

template <typename T, int NC, bool RES>
__global__ void __launch_bounds__(32 * LNF_WARPS, LNF_BLOCKS_PER_SM)
    ln_bwd_fused_kernel(const T* dy, const T* x, const float* mean,
                        const float* rstd, const T* g, T* __restrict__ dres,
                        int dres_init, int M, int d, float* __restrict__ part_ln, float* __restrict__ part_res) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  extern __shared__ float red[];  // [LNF_WARPS][3][d]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float sg[NC][VN], sb[NC][VN], sr[NC][VN];
#pragma unroll
  for (int k = 0; k < NC; ++k)
#pragma unroll
    for (int j = 0; j < VN; ++j) sg[k][j] = sb[k][j] = sr[k][j] = 0.f;
  // the rows stay packed (16-byte words) in registers and are unpacked on
  // each use, which leaves room to prefetch the next row (x, dy, the incoming
  // residual gradient, its mean and rstd) while this one is processed: two
  // rows of loads in flight per warp
  const int stride = gridDim.x * LNF_WARPS;
  int m = blockIdx.x * LNF_WARPS + warp;
  uint4 cx[NC], cd[NC], cr[NC];
  float cmu = 0.f, crs = 0.f;
  auto load_row = [&](int r, uint4 (&ux)[NC], uint4 (&ud)[NC], uint4 (&ur)[NC], float& mu_, float& rs_) {
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const int c = (lane + 32 * k) * VN;
      if (r < M && c < d) {
        ux[k] = *reinterpret_cast<const uint4*>(x + (long)r * d + c);
        ud[k] = *reinterpret_cast<const uint4*>(dy + (long)r * d + c);
        if (!dres_init) ur[k] = *reinterpret_cast<const uint4*>(dres + (long)r * d + c);
      }
    }
    if (r < M) {
      mu_ = mean[r];
      rs_ = rstd[r];
    }
  };
  load_row(m, cx, cd, cr, cmu, crs);
  for (; m < M; m += stride) {
    uint4 nx[NC], nd[NC], nr[NC];
    float nmu = 0.f, nrs = 0.f;
    load_row(m + stride, nx, nd, nr, nmu, nrs);
    const float mu = cmu, rs = crs;
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const int c = (lane + 32 * k) * VN;
      if (c < d) {
        float xv[VN], dv[VN], gv[VN];
        unpack16<T>(cx[k], xv);
        unpack16<T>(cd[k], dv);
        Vec<T>::load(g + c, gv);
#pragma unroll
        for (int j = 0; j < VN; ++j) {
          const float xh = (xv[j] - mu) * rs, gd = dv[j] * gv[j];
          s1 += gd;
          s2 += gd * xh;
          sg[k][j] += dv[j] * xh;
          sb[k][j] += dv[j];
        }
      }
    }
    s1 = warp_sum(s1) / d;
    s2 = warp_sum(s2) / d;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const int c = (lane + 32 * k) * VN;
      if (c < d) {
        float xv[VN], dv[VN], gv[VN], o[VN];
        unpack16<T>(cx[k], xv);
        unpack16<T>(cd[k], dv);
        Vec<T>::load(g + c, gv);
        if (!dres_init) {
          unpack16<T>(cr[k], o);
        } else {
#pragma unroll
          for (int j = 0; j < VN; ++j) o[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < VN; ++j) {
          const float xh = (xv[j] - mu) * rs, gd = dv[j] * gv[j];
          o[j] += rs * (gd - s1 - xh * s2);
          if (RES) sr[k][j] += o[j];
        }
        Vec<T>::store(dres + (long)m * d + c, o);
      }
    }
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      cx[k] = nx[k];
      cd[k] = nd[k];
      cr[k] = nr[k];
    }
    cmu = nmu;
    crs = nrs;
  }
  constexpr int NQ = RES ? 3 : 2;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * VN;
    if (c < d) {
#pragma unroll
      for (int j = 0; j < VN; ++j) {
        red[(warp * NQ + 0) * d + c + j] = sg[k][j];
        red[(warp * NQ + 1) * d + c + j] = sb[k][j];
        if (RES) red[(warp * NQ + 2) * d + c + j] = sr[k][j];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NQ * d; i += 32 * LNF_WARPS) {
    float t = red[i];
#pragma unroll
    for (int w = 1; w < LNF_WARPS; ++w) t += red[w * NQ * d + i];
    if (i < 2 * d)
      part_ln[(long)blockIdx.x * 2 * d + i] = t;
    else
      part_res[(long)blockIdx.x * d + (i - 2 * d)] = t;
  }
}

// bf16 rows of ln_bwd_fused_kernel with the arithmetic on fp32 pairs and
// gamma held in registers across a warp's rows.  Per element, in pairs:
//   xh = x rstd - mean rstd, gd = dy g, s1 += gd, s2 += gd xh,
//   dgamma += dy xh, dbeta += dy, then
//   dres = (init ? 0 : dres) + rstd (gd - s1/d - xh s2/d)   (and its column sum)
// Two blocks per SM (up to 255 registers a thread): the three column
// accumulators, gamma and two rows of loads stay in registers without spills.
constexpr int LNB_BLOCKS_PER_SM = 2;

template <int NC, bool RES>
__global__ void __launch_bounds__(32 * LNF_WARPS, LNB_BLOCKS_PER_SM)
    ln_bwd_bf16_kernel(const bf16* dy, const bf16* x, const float* mean,
                       const float* rstd, const bf16* g, bf16* __restrict__ dres,
                       int dres_init, int M, int d, float* __restrict__ part_ln, float* __restrict__ part_res) {
  pdl_start();
  extern __shared__ float red[];  // [LNF_WARPS][3][d]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float2 gg[NC][4];
  float2 sg[NC][4], sb[NC][4], sr[NC][4];
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * 8;
    const uint4 u = c < d ? *reinterpret_cast<const uint4*>(g + c) : make_uint4(0, 0, 0, 0);
    gg[k][0] = bf2w(u.x); gg[k][1] = bf2w(u.y); gg[k][2] = bf2w(u.z); gg[k][3] = bf2w(u.w);
#pragma unroll
    for (int j = 0; j < 4; ++j) sg[k][j] = sb[k][j] = sr[k][j] = make_float2(0.f, 0.f);
  }
  const float inv_d = 1.f / (float)d;
  const int stride = gridDim.x * LNF_WARPS;
  int m = blockIdx.x * LNF_WARPS + warp;
  uint4 cx[NC], cd[NC], cr[NC];
  float cmu = 0.f, crs = 0.f;
  auto load_row = [&](int r, uint4 (&ux)[NC], uint4 (&ud)[NC], uint4 (&ur)[NC], float& mu_, float& rs_) {
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const int c = (lane + 32 * k) * 8;
      if (r < M && c < d) {
        ux[k] = *reinterpret_cast<const uint4*>(x + (long)r * d + c);
        ud[k] = *reinterpret_cast<const uint4*>(dy + (long)r * d + c);
        ur[k] = dres_init ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4*>(dres + (long)r * d + c);
      } else {
        ux[k] = ud[k] = ur[k] = make_uint4(0, 0, 0, 0);
      }
    }
    if (r < M) {
      mu_ = mean[r];
      rs_ = rstd[r];
    }
  };
  load_row(m, cx, cd, cr, cmu, crs);
  for (; m < M; m += stride) {
    uint4 nx[NC], nd[NC], nr[NC];
    float nmu = 0.f, nrs = 0.f;
    load_row(m + stride, nx, nd, nr, nmu, nrs);
    const float2 rs2 = make_float2(crs, crs), c2 = make_float2(-cmu * crs, -cmu * crs);
    float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const uint32_t* xw = &cx[k].x;
      const uint32_t* dw = &cd[k].x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 dv = bf2w(dw[j]);
        const float2 xh = __ffma2_rn(bf2w(xw[j]), rs2, c2);
        const float2 gd = __fmul2_rn(dv, gg[k][j]);
        s1 = __fadd2_rn(s1, gd);
        s2 = __ffma2_rn(gd, xh, s2);
        sg[k][j] = __ffma2_rn(dv, xh, sg[k][j]);
        sb[k][j] = __fadd2_rn(sb[k][j], dv);
      }
    }
    const float m1 = warp_sum(s1.x + s1.y) * inv_d, m2 = warp_sum(s2.x + s2.y) * inv_d;
    const float2 nm1 = make_float2(-m1, -m1), nm2 = make_float2(-m2, -m2);
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const int c = (lane + 32 * k) * 8;
      const uint32_t* xw = &cx[k].x;
      const uint32_t* dw = &cd[k].x;
      const uint32_t* rw = &cr[k].x;
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 xh = __ffma2_rn(bf2w(xw[j]), rs2, c2);
        const float2 gd = __fmul2_rn(bf2w(dw[j]), gg[k][j]);
        const float2 t = __fadd2_rn(__ffma2_rn(xh, nm2, gd), nm1);   // gd - s1/d - xh s2/d
        const float2 o = __ffma2_rn(t, rs2, bf2w(rw[j]));
        if (RES) sr[k][j] = __fadd2_rn(sr[k][j], o);
        w[j] = pack_bf16x2(o.x, o.y);
      }
      if (c < d) *reinterpret_cast<uint4*>(dres + (long)m * d + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      cx[k] = nx[k];
      cd[k] = nd[k];
      cr[k] = nr[k];
    }
    cmu = nmu;
    crs = nrs;
  }
  constexpr int NQ = RES ? 3 : 2;
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    const int c = (lane + 32 * k) * 8;
    if (c < d) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        red[(warp * NQ + 0) * d + c + 2 * j] = sg[k][j].x;
        red[(warp * NQ + 0) * d + c + 2 * j + 1] = sg[k][j].y;
        red[(warp * NQ + 1) * d + c + 2 * j] = sb[k][j].x;
        red[(warp * NQ + 1) * d + c + 2 * j + 1] = sb[k][j].y;
        if (RES) {
          red[(warp * NQ + 2) * d + c + 2 * j] = sr[k][j].x;
          red[(warp * NQ + 2) * d + c + 2 * j + 1] = sr[k][j].y;
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NQ * d; i += 32 * LNF_WARPS) {
    float t = red[i];
#pragma unroll
    for (int w = 1; w < LNF_WARPS; ++w) t += red[w * NQ * d + i];
    if (i < 2 * d)
      part_ln[(long)blockIdx.x * 2 * d + i] = t;
    else
      part_res[(long)blockIdx.x * d + (i - 2 * d)] = t;
  }
}

// grad[j] = beta * grad[j] + sum_r part[r, j] (r ascending); 8 row slices per
// column reduced in a fixed order.
__global__ void reduce_rows_kernel(const float* part, int nrows, int n, float* __restrict__ grad,
                                   float beta) {
  pdl_start();
  __shared__ float sm[8][33];
  const int cx = threadIdx.x & 31, ry = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + cx;
  float s = 0.f;
  if (j < n)
    for (int r = ry; r < nrows; r += 8) s += part[(long)r * n + j];
  sm[ry][cx] = s;
  __syncthreads();
  if (ry == 0 && j < n) {
    float t = sm[0][cx];
    for (int k = 1; k < 8; ++k) t += sm[k][cx];
    grad[j] = (beta != 0.f ? beta * grad[j] : 0.f) + t;
  }
}

// The same reduction for up to MAX_REDUCE_JOBS (part, grad) pairs in one
// launch: block b takes a column block of the job whose column blocks
// contain b, 128 columns as four per thread (float4) when the job's width is
// a multiple of 4 and both arrays are 16-byte aligned, else 32 columns.
// Either way a column's sum runs over the same rows in the same order
// (thread row group ry takes rows ry, ry + 8, ... ascending, then the eight
// groups in order), so both forms give the same bits.
struct ReduceBatchArgs {
  ReduceJob job[MAX_REDUCE_JOBS];
  int start[MAX_REDUCE_JOBS + 1];  // first column block of each job
  int vec[MAX_REDUCE_JOBS];        // 1: float4 column blocks
  int njobs;
  float beta;
};

DEVI float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }

__global__ void reduce_rows_batch_kernel(const __grid_constant__ ReduceBatchArgs a) {
  pdl_start();
  __shared__ float4 sm4[8][32];
  float (*sm)[33] = reinterpret_cast<float (*)[33]>(&sm4[0][0]);  // the scalar form's [8][33]
  int jb = 0;
  while (jb + 1 < a.njobs && a.start[jb + 1] <= (int)blockIdx.x) ++jb;
  const float* part = a.job[jb].part;
  float* grad = a.job[jb].grad;
  const int nrows = a.job[jb].nrows, n = a.job[jb].n;
  const int cx = threadIdx.x & 31, ry = threadIdx.x >> 5;
  if (a.vec[jb]) {
    const int j = ((int)blockIdx.x - a.start[jb]) * 128 + 4 * cx;  // n % 4 == 0: all four inside or none
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < n) {
      int r = ry;
      // four rows in flight, added in row order
      for (; r + 24 < nrows; r += 32) {
        const float4 v0 = *reinterpret_cast<const float4*>(part + (long)r * n + j);
        const float4 v1 = *reinterpret_cast<const float4*>(part + (long)(r + 8) * n + j);
        const float4 v2 = *reinterpret_cast<const float4*>(part + (long)(r + 16) * n + j);
        const float4 v3 = *reinterpret_cast<const float4*>(part + (long)(r + 24) * n + j);
        s = add4(add4(add4(add4(s, v0), v1), v2), v3);
      }
      for (; r < nrows; r += 8) s = add4(s, *reinterpret_cast<const float4*>(part + (long)r * n + j));
    }
    sm4[ry][cx] = s;
    __syncthreads();
    if (ry == 0 && j < n) {
      float4 t = sm4[0][cx];
      for (int k = 1; k < 8; ++k) t = add4(t, sm4[k][cx]);
      float4* g4 = reinterpret_cast<float4*>(grad + j);
      const float4 old = a.beta != 0.f ? *g4 : make_float4(0.f, 0.f, 0.f, 0.f);
      *g4 = make_float4((a.beta != 0.f ? a.beta * old.x : 0.f) + t.x, (a.beta != 0.f ? a.beta * old.y : 0.f) + t.y,
                        (a.beta != 0.f ? a.beta * old.z : 0.f) + t.z, (a.beta != 0.f ? a.beta * old.w : 0.f) + t.w);
    }
    return;
  }
  const int j = ((int)blockIdx.x - a.start[jb]) * 32 + cx;
  float s = 0.f;
  if (j < n)
    for (int r = ry; r < nrows; r += 8) s += part[(long)r * n + j];
  sm[ry][cx] = s;
  __syncthreads();
  if (ry == 0 && j < n) {
    float t = sm[0][cx];
    for (int k = 1; k < 8; ++k) t += sm[k][cx];
    grad[j] = (a.beta != 0.f ? a.beta * grad[j] : 0.f) + t;
  }
}

// Column sums of x[M, N] over blocks of 128 rows -> part[rowblock, N].
constexpr int CS_ROWS = 128;

template <typename T>
__global__ void __launch_bounds__(256) colsum_kernel(const T* x, int M, int N,
                                                     float* __restrict__ part) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  __shared__ float red[8][32 * VN];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = (blockIdx.x * 32 + lane) * VN;
  const int r0 = blockIdx.y * CS_ROWS;
  float s[VN];
#pragma unroll
  for (int j = 0; j < VN; ++j) s[j] = 0.f;
  if (c < N) {
    for (int r = r0 + warp; r < min(r0 + CS_ROWS, M); r += 8) {
      float f[VN];
      Vec<T>::load(x + (long)r * N + c, f);
#pragma unroll
      for (int j = 0; j < VN; ++j) s[j] += f[j];
    }
  }
#pragma unroll
  for (int j = 0; j < VN; ++j) red[warp][lane * VN + j] = s[j];
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * VN; i += 256) {
    const int col = blockIdx.x * 32 * VN + i;
    if (col < N) {
      float t = red[0][i];
      for (int w = 1; w < 8; ++w) t += red[w][i];
      part[(long)blockIdx.y * N + col] = t;
    }
  }
}

// ---------------------------------------------------------- cross-entropy --
// Number of positions with a target (target -1 = masked); any other id outside
// [0, vocab_real) raises the token-range bit and counts as masked.
__global__ void __launch_bounds__(1024) count_targets_kernel(const int32_t* tgt, int M,
                                                             int vocab_real, int* __restrict__ n_valid, int* err) {
  pdl_start();
  __shared__ int red[32];
  int c = 0;
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    const int t = tgt[i];
    if (t >= 0 && t < vocab_real)
      ++c;
    else if (t != -1)
      atomicOr(err, DEV_ERR_TOKEN);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    *n_valid = t;
  }
}

// Row m: lse = log sum_v exp(z_v) over all V (padded) ids; loss = lse - z[y];
// then, in place, dz_v = exp(z_v - lse) - [v == y] (unscaled; the backward
// GEMMs apply grad_scale / M).
template <typename T>
__global__ void __launch_bounds__(256) ce_kernel(T* __restrict__ logits, const int32_t* tgt,
                                                 float* __restrict__ loss_rows, int V, int vocab_real,
                                                 const int* n_valid, int* err) {
  pdl_start();
  constexpr int VN = Vec<T>::N;
  constexpr int U = 4;  // 16-byte vectors in flight per thread and trip
  constexpr float L2E = 1.4426950408889634f;
  __shared__ float sm_m[8], sm_s[8];
  const int m = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  T* z = logits + (long)m * V;
  const int step = 256 * VN;
  if (tgt[m] == -1) {
    // masked position: no loss, and its dlogits row is zero
    if (threadIdx.x == 0) loss_rows[m] = 0.f;
    float zero[VN];
#pragma unroll
    for (int j = 0; j < VN; ++j) zero[j] = 0.f;
    for (int c = threadIdx.x * VN; c < V; c += step) Vec<T>::store(z + c, zero);
    return;
  }
  // pass 1: running maximum and sum of exp(z - max), U vectors per trip so the
  // loads of a trip overlap (V is a multiple of 128, so vectors never straddle it)
  float mx = -INFINITY, sum = 0.f;
  for (int c0 = threadIdx.x * VN; c0 < V; c0 += U * step) {
    float f[U][VN];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * step;
      if (c < V) {
        Vec<T>::load(z + c, f[u]);
      } else {
#pragma unroll
        for (int j = 0; j < VN; ++j) f[u][j] = -INFINITY;
      }
    }
    float lm = mx;
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < VN; ++j) lm = fmaxf(lm, f[u][j]);
    // the first trip always holds a finite element, so lm is finite here
    sum *= ex2_approx((mx - lm) * L2E);
    mx = lm;
    const float ml = mx * L2E;
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < VN; ++j) sum += ex2_approx(fmaf(f[u][j], L2E, -ml));
  }
  // combine (max, sum) pairs: within the warp, then across the eight warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, mx, o), s2 = __shfl_xor_sync(0xffffffffu, sum, o);
    const float mm = fmaxf(mx, m2);
    // (a thread that saw no element, possible only for V < 2048, holds -inf, 0)
    sum = (mx == -INFINITY ? 0.f : sum * ex2_approx((mx - mm) * L2E)) +
          (m2 == -INFINITY ? 0.f : s2 * ex2_approx((m2 - mm) * L2E));
    mx = mm;
  }
  if (lane == 0) {
    sm_m[warp] = mx;
    sm_s[warp] = sum;
  }
  __syncthreads();
  float M0 = sm_m[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) M0 = fmaxf(M0, sm_m[w]);
  float S0 = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w)
    if (sm_m[w] != -INFINITY) S0 += sm_s[w] * ex2_approx((sm_m[w] - M0) * L2E);
  const float lse = M0 + logf(S0);
  int y = tgt[m];
  if (y < 0 || y >= vocab_real) {
    if (threadIdx.x == 0) atomicOr(err, DEV_ERR_TOKEN);
    y = 0;
  }
  const float zy = to_f(z[y]);
  __syncthreads();  // every thread has read z[y] before it is overwritten
  if (threadIdx.x == 0) loss_rows[m] = lse - zy;
  // pass 2: dz = (softmax(z) - onehot(y)) * M / n_valid, in place: the backward
  // GEMMs scale by grad_scale / M, so the loss is the mean over the positions
  // that have a target (the factor is exactly 1 without masking)
  const float ll = lse * L2E;
  const int nv = *n_valid;
  const float rs = (float)gridDim.x / (float)(nv > 0 ? nv : 1);
  for (int c0 = threadIdx.x * VN; c0 < V; c0 += U * step) {
    float f[U][VN];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u * step < V) Vec<T>::load(z + c0 + u * step, f[u]);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * step;
      if (c < V) {
#pragma unroll
        for (int j = 0; j < VN; ++j)
          f[u][j] = (ex2_approx(fmaf(f[u][j], L2E, -ll)) - (c + j == y ? 1.f : 0.f)) * rs;
        Vec<T>::store(z + c, f[u]);
      }
    }
  }
}

// loss = sum(loss_rows) / n_valid (masked rows hold 0), fixed-order tree;
// flags a non-finite result.
__global__ void loss_mean_kernel(const float* rows, int M, const int* n_valid,
                                 float* __restrict__ loss, int* err) {
  pdl_start();
  __shared__ float sm[1024];
  float s = 0.f;
  for (int i = threadIdx.x; i < M; i += 1024) s += rows[i];
  sm[threadIdx.x] = s;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if (threadIdx.x < o) sm[threadIdx.x] += sm[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int nv = *n_valid;
    float v = sm[0] / (float)(nv > 0 ? nv : 1);
    *loss = v;
    if (!isfinite(v)) atomicOr(err, DEV_ERR_NONFINITE);
  }
}

// Cross-entropy from the LM head's partials (the EPI_CE_FWD epilogue of the
// tied LM-head GEMM): for row m and part p of 128 vocabulary columns,
// pm[p*M+m] = max_v z and ps[p*M+m] = sum_v exp(z - pm); zt[m] = z[m, target];
// e[m, v] = bf16 exp(z - pm) for v in part p.
// ce_merge_kernel, per row:
//   lse_m = max_p pm + log sum_p ps exp(pm - max)       (the row's log-sum-exp)
//   loss_m = lse_m - zt[m] (0 where masked)
// 32 rows per block; the eight warps take every eighth part and their partial
// results meet in shared memory in a fixed order.
// ce_dz_kernel, in place over e:
//   e[m, v] <- (e[m, v] exp(pm - lse_m) - [v == target]) M / n_valid
// (0 where masked), i.e. dz = (softmax - onehot) scaled so that the backward
// GEMMs' alpha = grad_scale / M gives the mean over the positions with a
// target.  One block per token row, four 16-byte loads in flight per thread.
__global__ void __launch_bounds__(256) ce_merge_kernel(const float* pm, const float* ps,
                                                       const float* zt, const int32_t* tgt,
                                                       int M, int P, int vocab_real, float* __restrict__ lse_out,
                                                       float* __restrict__ loss_rows) {
  pdl_start();
  constexpr float L2E = 1.4426950408889634f;
  __shared__ float red[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 32 + lane;
  const bool in = m < M;
  float mx = -INFINITY;
  // (four parts' loads in flight; the running maximum and, below, the sum
  // take the parts in the same order as a plain loop)
  if (in)
#pragma unroll 4
    for (int p = warp; p < P; p += 8) mx = fmaxf(mx, pm[(long)p * M + m]);
  red[warp][lane] = mx;
  __syncthreads();
  float gm = red[0][lane];
#pragma unroll
  for (int w = 1; w < 8; ++w) gm = fmaxf(gm, red[w][lane]);
  __syncthreads();
  float sum = 0.f;
  if (in)
#pragma unroll 4
    for (int p = warp; p < P; p += 8) {
      const long i = (long)p * M + m;
      sum += ps[i] * ex2_approx((pm[i] - gm) * L2E);
    }
  red[warp][lane] = sum;
  __syncthreads();
  if (warp == 0 && in) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w][lane];
    const float lse = gm + logf(tot);
    const int y = tgt[m];
    const bool valid = y >= 0 && y < vocab_real;
    lse_out[m] = lse;
    loss_rows[m] = valid ? lse - zt[m] : 0.f;
  }
}

__global__ void __launch_bounds__(256) ce_dz_kernel(bf16* __restrict__ e, const float* pm,
                                                    const float* lse, const int32_t* tgt,
                                                    int M, int V, int vocab_real, const int* n_valid) {
  pdl_start();
  constexpr float L2E = 1.4426950408889634f;
  constexpr int U = 4;
  const int m = blockIdx.x;
  const int y = tgt[m];
  const bool valid = y >= 0 && y < vocab_real;
  const int nv = *n_valid;
  const float full = (float)M / (float)(nv > 0 ? nv : 1);
  const float scale = valid ? full : 0.f;
  const float l2 = lse[m] * L2E;
  const int yv = valid ? y : -1;
  bf16* row = e + (long)m * V;
  const int pieces = V / 8;
  // the row's per-part scales exp(pm - lse) * scale, once, in shared memory
  extern __shared__ float part_scale[];  // [V / 128]
  for (int p = threadIdx.x; p < (V >> 7); p += 256)
    part_scale[p] = ex2_approx(fmaf(pm[(long)p * M + m], L2E, -l2)) * scale;
  __syncthreads();
  // the whole row, 16-byte pieces 4 KB apart, four loads in flight per thread
  for (int p0 = threadIdx.x; p0 < pieces; p0 += 256 * U) {
    uint4 u[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int pi = p0 + 256 * k;
      if (pi < pieces) u[k] = *reinterpret_cast<const uint4*>(row + 8 * pi);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int pi = p0 + 256 * k;
      if (pi < pieces) {
        const int c = 8 * pi;
        // (V is a multiple of 128: a 16-byte piece lies in one part)
        const float s = part_scale[c >> 7];
        const int dy = yv - c;
        float f[8] = {bf16lo(u[k].x), bf16hi(u[k].x), bf16lo(u[k].y), bf16hi(u[k].y),
                      bf16lo(u[k].z), bf16hi(u[k].z), bf16lo(u[k].w), bf16hi(u[k].w)};
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = f[j] * s - (dy == j ? full : 0.f);
        uint4 o;
        o.x = pack_bf16x2(f[0], f[1]);
        o.y = pack_bf16x2(f[2], f[3]);
        o.z = pack_bf16x2(f[4], f[5]);
        o.w = pack_bf16x2(f[6], f[7]);
        *reinterpret_cast<uint4*>(row + c) = o;
      }
    }
  }
}

// ---------------------------------------------------------------- AdamW --

// Which flat-layout elements are 2-D weights (wte, wpe, w_qkv, w_o, w_fc,
// w_mp): those get weight decay and, at init, N(0, std) draws.
// Returns 0 = 1-D tensor, 1 = 2-D weight, 2 = residual projection (w_o, w_mp);
// *one = 1 for LayerNorm gains.
DEVI int tensor_kind(long i, const LayoutDims& L, int* one) {
  const long d = L.d;
  *one = 0;
  const long emb = (L.V + L.T) * d;
  if (i < emb) return 1;
  const long per = 12 * d * d + 13 * d;
  const long j = i - emb;
  if (j >= L.L * per) {  // lnf_g, lnf_b
    *one = (j - L.L * per) < d;
    return 0;
  }
  const long r = j % per;
  long o = d;
  if (r < o) { *one = 1; return 0; }  // ln1_g
  o += d;
  if (r < o) return 0;                // ln1_b
  o += 3 * d * d;
  if (r < o) return 1;                // w_qkv
  o += 3 * d;
  if (r < o) return 0;                // b_qkv
  o += d * d;
  if (r < o) return 2;                // w_o
  o += d;
  if (r < o) return 0;                // b_o
  o += d;
  if (r < o) { *one = 1; return 0; }  // ln2_g
  o += d;
  if (r < o) return 0;                // ln2_b
  o += 4 * d * d;
  if (r < o) return 1;                // w_fc
  o += 4 * d;
  if (r < o) return 0;                // b_fc
  o += 4 * d * d;
  if (r < o) return 2;                // w_mp
  return 0;                           // b_mp
}

// Global L2 norm of the flat gradient in two fixed-order passes: per-block
// sums of squares over a grid of GRAD_NORM_PARTS blocks (fixed, so the result
// does not depend on the device), then one block adds them and takes the root.
__global__ void __launch_bounds__(256) sumsq_kernel(const float* g, long n4, float* __restrict__ part) {
  pdl_start();
  __shared__ float red[8];
  float s = 0.f;
  for (long i4 = blockIdx.x * (long)blockDim.x + threadIdx.x; i4 < n4; i4 += (long)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(g)[i4];
    s += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < 8; ++w) t += red[w];
    part[blockIdx.x] = t;
  }
}

__global__ void __launch_bounds__(256) norm_final_kernel(const float* part, int nparts,
                                                         float* __restrict__ norm) {
  pdl_start();
  __shared__ float red[8];
  float s = 0.f;
  for (int i = threadIdx.x; i < nparts; i += 256) s += part[i];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < 8; ++w) t += red[w];
    *norm = sqrtf(t);
  }
}

// With gnorm != NULL the gradient is first scaled by min(1, max_norm / (gnorm + 1e-6))
// (global-norm clipping).
// Elements [base, base + 4 n4) of the flat buffers; the pointers point at
// element base, whose layout position decides the weight-decay mask.
__global__ void adamw_kernel(float* __restrict__ p, const float* g, float* __restrict__ m,
                             float* __restrict__ v, uint16_t* __restrict__ shadow, long n4, long base,
                             LayoutDims L, AdamArgs a, const float* gnorm, float max_norm) {
  pdl_start();
  float clip = 1.f;
  if (gnorm) {
    const float c = max_norm / (*gnorm + 1e-6f);
    clip = c < 1.f ? c : 1.f;
  }
  for (long i4 = blockIdx.x * (long)blockDim.x + threadIdx.x; i4 < n4; i4 += (long)gridDim.x * blockDim.x) {
    const long i = base + i4 * 4;
    int one;
    const bool decay = tensor_kind(i, L, &one) != 0;
    float4 pp = reinterpret_cast<float4*>(p)[i4];
    float4 gg = reinterpret_cast<const float4*>(g)[i4];
    gg.x *= clip; gg.y *= clip; gg.z *= clip; gg.w *= clip;
    float4 mm = reinterpret_cast<float4*>(m)[i4];
    float4 vv = reinterpret_cast<float4*>(v)[i4];
    const float dec = decay ? 1.f - a.lr * a.wd : 1.f;
    float* P = &pp.x;
    const float* G = &gg.x;
    float* Mm = &mm.x;
    float* Vv = &vv.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      Mm[j] = a.beta1 * Mm[j] + (1.f - a.beta1) * G[j];
      Vv[j] = a.beta2 * Vv[j] + (1.f - a.beta2) * G[j] * G[j];
      const float mh = Mm[j] / a.bc1;
      const float vh = Vv[j] / a.bc2;
      P[j] = P[j] * dec - a.lr * mh / (sqrtf(vh) + a.eps);
    }
    reinterpret_cast<float4*>(p)[i4] = pp;
    reinterpret_cast<float4*>(m)[i4] = mm;
    reinterpret_cast<float4*>(v)[i4] = vv;
    if (shadow) {
      uint2 u = make_uint2(pack_bf16x2(pp.x, pp.y), pack_bf16x2(pp.z, pp.w));
      reinterpret_cast<uint2*>(shadow)[i4] = u;
    }
  }
}

// --------------------------------------------------------- initialisation --
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw: "Parallel random numbers: as easy
// as 1, 2, 3", SC'11): 10 rounds of two 32x32->64 multiplies with a Weyl key
// schedule; counter = element index, key = seed.
DEVI void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c[0], hi0 = __umulhi(0xD2511F53u, c[0]);
    const uint32_t lo1 = 0xCD9E8D57u * c[2], hi1 = __umulhi(0xCD9E8D57u, c[2]);
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

__global__ void init_kernel(float* __restrict__ p, long n, LayoutDims L, uint64_t seed) {
  pdl_start();
  const float std_w = 0.02f;
  const float std_proj = 0.02f / sqrtf(2.f * (float)L.L);
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    int one;
    const int kind = tensor_kind(i, L, &one);
    float val;
    if (kind == 0) {
      val = one ? 1.f : 0.f;
    } else {
      uint32_t c[4] = {(uint32_t)i, (uint32_t)((uint64_t)i >> 32), 0u, 0u};
      philox4x32_10(c, (uint32_t)seed, (uint32_t)(seed >> 32));
      // Box-Muller on two uniforms in (0, 1]
      const float u1 = ((float)c[0] + 1.f) * 2.3283064365386963e-10f;
      const float u2 = (float)c[1] * 2.3283064365386963e-10f;
      const float z = sqrtf(-2.f * logf(fminf(u1, 1.f))) * cospif(2.f * u2);
      val = z * (kind == 2 ? std_proj : std_w);
    }
    p[i] = val;
  }
}

__global__ void cast_shadow_kernel(const float* p, uint16_t* __restrict__ s, long n4) {
  pdl_start();
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
    float4 v = reinterpret_cast<const float4*>(p)[i];
    reinterpret_cast<uint2*>(s)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

int grid_for(long n, int threads) {
  long b = (n + threads - 1) / threads;
  long cap = (long)num_sms() * 16;
  return (int)(b < cap ? (b < 1 ? 1 : b) : cap);
}

template <typename T, int NC>
int ln_fwd_launch(const void* x, const void* g, const void* b, void* y, float* mean, float* rstd, int M,
                   int d, cudaStream_t st) {
  // (a packed-arithmetic bf16 variant with gamma / beta in registers over
  // four rows per warp measured the same in the step and 13 % slower at
  // 131072 rows: this kernel is not issue-bound enough for it to pay)
  CUDA_TRY(launch_k(ln_fwd_kernel<T, NC>, (M + 7) / 8, 256, 0, st,
      (const T*)x, (const T*)g, (const T*)b, (T*)y, mean, rstd, M, d));
  return GPT2_OK;
}

template <typename T>
int ln_fwd_dispatch(const void* x, const void* g, const void* b, void* y, float* mean, float* rstd, int M,
                    int d, cudaStream_t st) {
  const int nc = (d / Vec<T>::N + 31) / 32;
  int rc = GPT2_OK;
  switch (nc) {
    case 1: rc = ln_fwd_launch<T, 1>(x, g, b, y, mean, rstd, M, d, st); break;
    case 2: rc = ln_fwd_launch<T, 2>(x, g, b, y, mean, rstd, M, d, st); break;
    case 3: rc = ln_fwd_launch<T, 3>(x, g, b, y, mean, rstd, M, d, st); break;
    case 4: rc = ln_fwd_launch<T, 4>(x, g, b, y, mean, rstd, M, d, st); break;
    case 5: rc = ln_fwd_launch<T, 5>(x, g, b, y, mean, rstd, M, d, st); break;
    case 6: rc = ln_fwd_launch<T, 6>(x, g, b, y, mean, rstd, M, d, st); break;
    case 7: rc = ln_fwd_launch<T, 7>(x, g, b, y, mean, rstd, M, d, st); break;
    case 8: rc = ln_fwd_launch<T, 8>(x, g, b, y, mean, rstd, M, d, st); break;
    default: return GPT2_ERR_UNSUPPORTED_SHAPE;
  }
  if (rc) return rc;
  LAUNCH_CHECK();
  return GPT2_OK;
}

int ln_fused_blocks(int M, int per_sm = LNF_BLOCKS_PER_SM) {
  const int b = per_sm * num_sms();
  const int need = (M + LNF_WARPS - 1) / LNF_WARPS;
  return b < need ? b : need;
}

// The fused one-pass kernel keeps 2-3 column accumulators per element a lane
// owns, so it is used while a lane owns at most 24 columns of the row (d 768
// in bf16 or fp32); wider rows take the row kernel plus the column-sum
// kernels.
template <typename T, int NC>
int ln_bwd_launch(const void* dy, const void* x, const float* mean, const float* rstd, const void* g,
                   void* dres, int init, float* part, float* part_res, int* nblk, int M, int d, cudaStream_t st) {
  constexpr int VN = Vec<T>::N;
  if constexpr (NC * VN <= 24) {
    const bool pk = std::is_same<T, bf16>::value;
    const int blocks = ln_fused_blocks(M, pk ? LNB_BLOCKS_PER_SM : LNF_BLOCKS_PER_SM);
    *nblk = blocks;
    if constexpr (std::is_same<T, bf16>::value) {
      if (part_res) {
        const size_t smem = (size_t)LNF_WARPS * 3 * d * sizeof(float);
        CUDA_TRY(launch_k(ln_bwd_bf16_kernel<NC, true>, blocks, 32 * LNF_WARPS, smem, st, (const bf16*)dy,
                          (const bf16*)x, mean, rstd, (const bf16*)g, (bf16*)dres, init, M, d, part, part_res));
      } else {
        const size_t smem = (size_t)LNF_WARPS * 2 * d * sizeof(float);
        CUDA_TRY(launch_k(ln_bwd_bf16_kernel<NC, false>, blocks, 32 * LNF_WARPS, smem, st, (const bf16*)dy,
                          (const bf16*)x, mean, rstd, (const bf16*)g, (bf16*)dres, init, M, d, part, nullptr));
      }
      return GPT2_OK;
    }
    if (part_res) {
      const size_t smem = (size_t)LNF_WARPS * 3 * d * sizeof(float);
      CUDA_TRY(launch_k(ln_bwd_fused_kernel<T, NC, true>, blocks, 32 * LNF_WARPS, smem, st, 
          (const T*)dy, (const T*)x, mean, rstd, (const T*)g, (T*)dres, init, M, d, part, part_res));
    } else {
      const size_t smem = (size_t)LNF_WARPS * 2 * d * sizeof(float);
      CUDA_TRY(launch_k(ln_bwd_fused_kernel<T, NC, false>, blocks, 32 * LNF_WARPS, smem, st, 
          (const T*)dy, (const T*)x, mean, rstd, (const T*)g, (T*)dres, init, M, d, part, nullptr));
    }
    return GPT2_OK;
  }
  *nblk = (M + LNP_ROWS - 1) / LNP_ROWS;
  CUDA_TRY(launch_k(ln_bwd_dx_kernel<T, NC>, (M + 7) / 8, 256, 0, st,
      (const T*)dy, (const T*)x, mean, rstd, (const T*)g, (T*)dres, init, M, d));
  gpt2_count_launch();
  dim3 grid((d + 32 * VN - 1) / (32 * VN), (M + LNP_ROWS - 1) / LNP_ROWS);
  CUDA_TRY(launch_k(ln_param_colsum_kernel<T>, grid, 256, 0, st, (const T*)dy, (const T*)x, mean, rstd, M, d, part));
  if (part_res) {
    gpt2_count_launch();
    // column sums of the new dres in the same row blocks (CS_ROWS == LNP_ROWS)
    dim3 g2((d + 32 * VN - 1) / (32 * VN), (M + CS_ROWS - 1) / CS_ROWS);
    CUDA_TRY(launch_k(colsum_kernel<T>, g2, 256, 0, st, (const T*)dres, M, d, part_res));
  }
  return GPT2_OK;
}

template <typename T>
int ln_bwd_dispatch(const void* dy, const void* x, const float* mean, const float* rstd, const void* g,
                    void* dres, int init, float* part, float* part_res, int* nblk, int M, int d, cudaStream_t st) {
  const int nc = (d / Vec<T>::N + 31) / 32;
  int rc = GPT2_OK;
  switch (nc) {
    case 1: rc = ln_bwd_launch<T, 1>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 2: rc = ln_bwd_launch<T, 2>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 3: rc = ln_bwd_launch<T, 3>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 4: rc = ln_bwd_launch<T, 4>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 5: rc = ln_bwd_launch<T, 5>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 6: rc = ln_bwd_launch<T, 6>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 7: rc = ln_bwd_launch<T, 7>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    case 8: rc = ln_bwd_launch<T, 8>(dy, x, mean, rstd, g, dres, init, part, part_res, nblk, M, d, st); break;
    default: return GPT2_ERR_UNSUPPORTED_SHAPE;
  }
  if (rc) return rc;
  LAUNCH_CHECK();
  return GPT2_OK;
}

}  // namespace

// ------------------------------------------------------------ launchers --

int embed_fwd(int f32, const int32_t* tok, const void* wte, const void* wpe, void* x, int M, int T, int d,
              int vocab_real, int* err, cudaStream_t st) {
  const int blocks = (M + 7) / 8;
  if (f32)
    CUDA_TRY(launch_k(embed_fwd_kernel<float>, blocks, 256, 0, st,
        tok, (const float*)wte, (const float*)wpe, (float*)x, M, T, d, vocab_real, err));
  else
    CUDA_TRY(launch_k(embed_fwd_kernel<bf16>, blocks, 256, 0, st,
        tok, (const bf16*)wte, (const bf16*)wpe, (bf16*)x, M, T, d, vocab_real, err));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int layernorm_fwd(int f32, const void* x, const void* g, const void* b, void* y, float* mean, float* rstd,
                  int M, int d, cudaStream_t st) {
  return f32 ? ln_fwd_dispatch<float>(x, g, b, y, mean, rstd, M, d, st)
             : ln_fwd_dispatch<bf16>(x, g, b, y, mean, rstd, M, d, st);
}

size_t layernorm_bwd_part_rows(int M) {
  const int a = ln_fused_blocks(M), b = (M + LNP_ROWS - 1) / LNP_ROWS;
  return (size_t)(a > b ? a : b);
}
size_t layernorm_bwd_part_floats(int M, int d) { return layernorm_bwd_part_rows(M) * 2 * d; }

int layernorm_bwd(int f32, const void* dy, const void* x, const float* mean, const float* rstd, const void* g,
                  void* dres, int dres_init, float* part, float* part_res, int* nblk, int M, int d,
                  cudaStream_t st) {
  return f32 ? ln_bwd_dispatch<float>(dy, x, mean, rstd, g, dres, dres_init, part, part_res, nblk, M, d, st)
             : ln_bwd_dispatch<bf16>(dy, x, mean, rstd, g, dres, dres_init, part, part_res, nblk, M, d, st);
}

int reduce_rows_f32(const float* part, int nrows, int n, float* grad, float beta, cudaStream_t st) {
  CUDA_TRY(launch_k(reduce_rows_kernel, (n + 31) / 32, 256, 0, st, part, nrows, n, grad, beta));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int reduce_rows_batch(const ReduceJob* jobs, int njobs, float beta, cudaStream_t st) {
  for (int j0 = 0; j0 < njobs; j0 += MAX_REDUCE_JOBS) {
    ReduceBatchArgs a;
    a.njobs = njobs - j0 < MAX_REDUCE_JOBS ? njobs - j0 : MAX_REDUCE_JOBS;
    a.beta = beta;
    int blocks = 0;
    for (int k = 0; k < a.njobs; ++k) {
      const ReduceJob& jk = jobs[j0 + k];
      a.job[k] = jk;
      a.start[k] = blocks;
      a.vec[k] = jk.n % 4 == 0 && reinterpret_cast<uintptr_t>(jk.part) % 16 == 0 &&
                 reinterpret_cast<uintptr_t>(jk.grad) % 16 == 0;
      blocks += a.vec[k] ? (jk.n + 127) / 128 : (jk.n + 31) / 32;
    }
    a.start[a.njobs] = blocks;
    if (blocks == 0) continue;
    CUDA_TRY(launch_k(reduce_rows_batch_kernel, blocks, 256, 0, st, a));
    LAUNCH_CHECK();
  }
  return GPT2_OK;
}

size_t colsum_part_floats(int M, int N) { return (size_t)((M + CS_ROWS - 1) / CS_ROWS) * N; }

int colsum_partial(int f32, const void* x, int M, int N, float* part, int* nblk, cudaStream_t st) {
  *nblk = (M + CS_ROWS - 1) / CS_ROWS;
  const int vn = f32 ? 4 : 8;
  dim3 grid((N + 32 * vn - 1) / (32 * vn), *nblk);
  if (f32)
    CUDA_TRY(launch_k(colsum_kernel<float>, grid, 256, 0, st, (const float*)x, M, N, part));
  else
    CUDA_TRY(launch_k(colsum_kernel<bf16>, grid, 256, 0, st, (const bf16*)x, M, N, part));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int count_targets(const int32_t* tgt, int M, int vocab_real, int* n_valid, int* err, cudaStream_t st) {
  CUDA_TRY(launch_k(count_targets_kernel, 1, 1024, 0, st, tgt, M, vocab_real, n_valid, err));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int ce_fwd(int f32, void* logits, const int32_t* tgt, float* loss_rows, int M, int V, int vocab_real,
           const int* n_valid, int* err, cudaStream_t st) {
  if (f32)
    CUDA_TRY(launch_k(ce_kernel<float>, M, 256, 0, st, (float*)logits, tgt, loss_rows, V, vocab_real, n_valid,
                      err));
  else
    CUDA_TRY(launch_k(ce_kernel<bf16>, M, 256, 0, st, (bf16*)logits, tgt, loss_rows, V, vocab_real, n_valid,
                      err));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int ce_merge_dz(const float* part_max, const float* part_sum, const float* zt, const int32_t* tgt, void* e,
                float* lse, int M, int V, int vocab_real, const int* n_valid, float* loss_rows, cudaStream_t st) {
  if (V % 128) return GPT2_ERR_UNSUPPORTED_SHAPE;
  CUDA_TRY(launch_k(ce_merge_kernel, (M + 31) / 32, 256, 0, st, part_max, part_sum, zt, tgt, M, V / 128, vocab_real,
                    lse, loss_rows));
  LAUNCH_CHECK();
  CUDA_TRY(launch_k(ce_dz_kernel, M, 256, (size_t)(V / 128) * sizeof(float), st, (bf16*)e, part_max,
                    (const float*)lse, tgt, M, V, vocab_real, n_valid));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int loss_mean(const float* loss_rows, int M, const int* n_valid, float* loss, int* err, cudaStream_t st) {
  CUDA_TRY(launch_k(loss_mean_kernel, 1, 1024, 0, st, loss_rows, M, n_valid, loss, err));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int embed_bwd(int f32, const int32_t* tok, const void* dx, float* dwte, float* dwpe, long long* acc,
              uint8_t* touched, int M, int T, int d, int V, int wpe_accumulate, float grad_scale, cudaStream_t st) {
  const long n = (long)M * d;
  unsigned long long* a = reinterpret_cast<unsigned long long*>(acc);
  const double gs = fabs((double)grad_scale);
  const double fix = FIX_SCALE / (gs > 0.0 && gs < 1e30 ? gs : 1.0);
  if (f32)
    CUDA_TRY(launch_k(embed_scatter_kernel<float>, (unsigned)((n + 255) / 256), 256, 0, st,
        tok, (const float*)dx, a, touched, M, d, V, fix));
  else
    CUDA_TRY(launch_k(embed_scatter_kernel<bf16>, (unsigned)((n + 255) / 256), 256, 0, st,
        tok, (const bf16*)dx, a, touched, M, d, V, fix));
  LAUNCH_CHECK();
  CUDA_TRY(launch_k(embed_convert_kernel, (V + 7) / 8, 256, 0, st, a, touched, dwte, V, d, 1.0 / fix));
  LAUNCH_CHECK();
  const long tn = (long)T * d;
  const int B = M / T;
  const int vn = f32 ? 4 : 8;
  const bool vec = tn % vn == 0 && reinterpret_cast<uintptr_t>(dx) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(dwpe) % 16 == 0;
  if (vec && f32)
    CUDA_TRY(launch_k(wpe_grad_vec_kernel<float>, (unsigned)((tn / vn + 255) / 256), 256, 0, st,
        (const float*)dx, dwpe, B, tn, wpe_accumulate));
  else if (vec)
    CUDA_TRY(launch_k(wpe_grad_vec_kernel<bf16>, (unsigned)((tn / vn + 255) / 256), 256, 0, st,
        (const bf16*)dx, dwpe, B, tn, wpe_accumulate));
  else if (f32)
    CUDA_TRY(launch_k(wpe_grad_kernel<float>, (unsigned)((tn + 255) / 256), 256, 0, st,
        (const float*)dx, dwpe, B, T, d, wpe_accumulate));
  else
    CUDA_TRY(launch_k(wpe_grad_kernel<bf16>, (unsigned)((tn + 255) / 256), 256, 0, st, (const bf16*)dx, dwpe, B, T, d,
                                                                        wpe_accumulate));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int grad_norm(const float* g, size_t n, float* part, float* norm, cudaStream_t st) {
  if (n % 4) return GPT2_ERR_UNSUPPORTED_SHAPE;
  CUDA_TRY(launch_k(sumsq_kernel, GRAD_NORM_PARTS, 256, 0, st, g, (long)(n / 4), part));
  LAUNCH_CHECK();
  CUDA_TRY(launch_k(norm_final_kernel, 1, 256, 0, st, (const float*)part, GRAD_NORM_PARTS, norm));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int adamw(float* p, const float* g, float* m, float* v, uint16_t* shadow, size_t n, const LayoutDims& ld,
          const AdamArgs& a, const float* gnorm, float max_norm, cudaStream_t st, size_t base) {
  const long n4 = (long)(n / 4);
  if (n4 == 0) return GPT2_OK;
  CUDA_TRY(launch_k(adamw_kernel, grid_for(n4, 256), 256, 0, st, p + base, g + base, m + base, v + base,
                    shadow ? shadow + base : nullptr, n4, (long)base, ld, a, gnorm, max_norm));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int init_params(float* p, size_t n, const LayoutDims& ld, uint64_t seed, cudaStream_t st) {
  CUDA_TRY(launch_k(init_kernel, grid_for((long)n, 256), 256, 0, st, p, (long)n, ld, seed));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int cast_shadow(const float* p, uint16_t* shadow, size_t n, cudaStream_t st) {
  const long n4 = (long)(n / 4);
  CUDA_TRY(launch_k(cast_shadow_kernel, grid_for(n4, 256), 256, 0, st, p, shadow, n4));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int fill_zero(void* p, size_t bytes, cudaStream_t st) {
  CUDA_TRY(cudaMemsetAsync(p, 0, bytes, st));
  return GPT2_OK;
}
