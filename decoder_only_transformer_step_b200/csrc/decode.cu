// Incremental decoding with a key/value cache: the inference forward of the
// sampling loop ("Criei GPT-2 do zero com uma RTX 4090", sections "Vendo o
// modelo ficar mais inteligente aos poucos" and "Conversando de verdade com
// ele": the model continues a prompt one token at a time).
//
// One decode step feeds one token per sequence.  At a handful of rows every
// weight matrix is read once per step and used for only `rows` dot products,
// so the step is bound by HBM reads of the weights (plus the cache), not by
// tensor-core throughput: the matrix products here are CUDA-core GEMVs that
// stream each weight row once with 16-byte non-allocating loads, reuse it for
// all rows held in shared memory, and fuse the LayerNorm in front of them and
// the bias / GELU / residual / cache write behind them.  Attention of the new
// query against the cached keys and values runs one block per (head, row).
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr int GV_WARPS = 8;  // warps per GEMV block
constexpr int GV_COLS = 4;   // output columns per warp and pass
constexpr int LN_MAX_K = 2048;  // widest LayerNorm'd input row (d_model)
constexpr int GV_CHUNK = 4;     // k iterations whose weight loads are in flight together
constexpr int GV_STAGE = 16;    // input loads in flight per thread while staging

// 16 bytes of T as fp32
template <typename T> struct V16;
template <> struct V16<bf16> {
  static constexpr int N = 8;
  DEVI static void unpack(const uint4& u, float* f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
  }
};
template <> struct V16<float> {
  static constexpr int N = 4;
  DEVI static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};

// Four consecutive T as fp32.
DEVI float4 ld4f(const bf16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
}
DEVI float4 ld4f(const float* p) { return *reinterpret_cast<const float4*>(p); }

// Weights are read once per step: keep them out of L1.  Volatile, with a
// memory clobber, so that each load stays on the side of the kernel's
// grid-dependency wait where the code puts it (a plain asm is free to move).
DEVI uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p)
               : "memory");
  return r;
}

// Sums each of the P values of v over the 32 lanes, halving the values a lane
// holds at every exchange (lanes whose bit O is set keep the upper half); a
// step with one value left is a plain butterfly add.  Afterwards v[j] of lane
// l is the total of index rs_index(l, j).
template <int CNT, int O> struct ReduceScatter {
  template <int P> DEVI static void run(float (&v)[P], int lane) {
    if constexpr (O > 0) {
      if constexpr (CNT > 1) {
        constexpr int H = CNT / 2;
        const bool up = (lane & O) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = up ? v[i] : v[i + H];
          const float keep = up ? v[i + H] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
        }
        ReduceScatter<H, O / 2>::run(v, lane);
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
        ReduceScatter<1, O / 2>::run(v, lane);
      }
    }
  }
};
// Index of the total in v[j] of lane l; *owner is false for all but one of
// the lanes holding copies of the same total.
template <int P> DEVI int rs_index(int lane, int j, bool* owner) {
  int idx = j, cnt = P;
  bool own = true;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (cnt > 1) {
      cnt >>= 1;
      if (lane & o) idx += cnt;
    } else if (lane & o) {
      own = false;
    }
  }
  *owner = own;
  return idx;
}

// DECODE_QKV: + bias; q -> out (fp32), k and v -> the cache at pos[r]
// DECODE_RESID: out[r, n] += acc + bias[n] (the fp32 residual stream)
// DECODE_GELU: out[r, n] = GELU(acc + bias[n]);  DECODE_LOGITS: out[r, n] = acc
constexpr int DEC_QKV = DECODE_QKV, DEC_RESID = DECODE_RESID, DEC_GELU = DECODE_GELU, DEC_LOGITS = DECODE_LOGITS;

struct GemvArgs {
  const void* in;    // [rows, K] (row pitch K): fp32, or T when in_t
  int in_t;
  const void* W;     // T [N, K]
  const void* bias;  // T [N] (not DEC_LOGITS)
  const void* ln_g;  // T [K] (LayerNorm in front)
  const void* ln_b;
  void* out;         // [rows, ldo]: T for DEC_GELU, else fp32
  long ldo;
  int rows, N, K;
  // DEC_QKV: this layer's K and V planes [rows][H][max_len][hd]
  void* kc;
  void* vc;
  const int32_t* pos;
  int d, H, hd, max_len;
};

// Mean and 1/sqrt(var + 1e-5) (biased variance) of a row held as NC float4
// pieces per lane (pieces at or past K4 are zero and not counted).
template <int NC>
DEVI void ln_stats(const float4 (&v)[NC], int lane, int K4, int K, float* mu, float* rs) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < NC; ++c) s += (v[c].x + v[c].y) + (v[c].z + v[c].w);
  const float m = warp_sum(s) / K;
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    if (lane + 32 * c < K4) {
      const float t0 = v[c].x - m, t1 = v[c].y - m, t2 = v[c].z - m, t3 = v[c].w - m;
      q += (t0 * t0 + t1 * t1) + (t2 * t2 + t3 * t3);
    }
  }
  *mu = m;
  *rs = rsqrtf(warp_sum(q) / K + 1e-5f);
}
template <typename T>
DEVI void ln_store4(T* dst, float4 x, float4 g, float4 b, float mu, float rs) {
  dst[0] = from_f<T>((x.x - mu) * rs * g.x + b.x);
  dst[1] = from_f<T>((x.y - mu) * rs * g.y + b.y);
  dst[2] = from_f<T>((x.z - mu) * rs * g.z + b.z);
  dst[3] = from_f<T>((x.w - mu) * rs * g.w + b.w);
}

// Input rows -> shared memory as T, row pitch ld elements (rows past a.rows
// zero).  Every load of a row is issued before the first use (one memory
// round trip per row): 16-byte loads, the LayerNorm's row held in registers
// for its two statistics.  nw warps take the rows of the LayerNorm.
template <typename T, int ROWS, bool LN>
DEVI void gemv_stage_rows(const GemvArgs& a, T* xs, int ld, int warp, int lane, int nw) {
  const int K = a.K;
  constexpr int VN = V16<T>::N;
  if constexpr (LN) {
    constexpr int NC = LN_MAX_K / 128;  // float4 pieces per lane (widest row)
    constexpr int NC_FAST = 8;          // rows up to 1024 wide
    const T* g = reinterpret_cast<const T*>(a.ln_g);
    const T* b = reinterpret_cast<const T*>(a.ln_b);
    const int K4 = K / 4;
    for (int r = warp; r < ROWS; r += nw) {
      T* dst = xs + (size_t)r * ld;
      if (r >= a.rows) {
        for (int k = lane; k < K; k += 32) dst[k] = from_f<T>(0.f);
        continue;
      }
      const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.in) + (size_t)r * K);
      if (K4 <= 32 * NC_FAST) {
        // the row and its gains and shifts in one round trip
        float4 v[NC_FAST], gv[NC_FAST], bv[NC_FAST];
#pragma unroll
        for (int c = 0; c < NC_FAST; ++c) {
          const int i = lane + 32 * c;
          const bool in = i < K4;
          v[c] = in ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
          gv[c] = in ? ld4f(g + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
          bv[c] = in ? ld4f(b + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mu, rs;
        ln_stats<NC_FAST>(v, lane, K4, K, &mu, &rs);
#pragma unroll
        for (int c = 0; c < NC_FAST; ++c) {
          const int i = lane + 32 * c;
          if (i < K4) ln_store4(dst + 4 * i, v[c], gv[c], bv[c], mu, rs);
        }
      } else {
        // wide rows: the row in registers, gains and shifts a few pieces at a time
        float4 v[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const int i = lane + 32 * c;
          v[c] = i < K4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mu, rs;
        ln_stats<NC>(v, lane, K4, K, &mu, &rs);
#pragma unroll 4
        for (int c = 0; c < NC; ++c) {
          const int i = lane + 32 * c;
          if (i < K4) ln_store4(dst + 4 * i, v[c], ld4f(g + 4 * i), ld4f(b + 4 * i), mu, rs);
        }
      }
    }
  } else if (a.in_t) {
    // rows already in T: 16-byte copies, GV_STAGE of them in flight per thread
    const int KV = K / VN, n16 = ROWS * KV, nthr = nw * 32;
    const uint4* src = reinterpret_cast<const uint4*>(a.in);
    for (int i0 = threadIdx.x; i0 < n16; i0 += GV_STAGE * nthr) {
      uint4 v[GV_STAGE];
#pragma unroll
      for (int u = 0; u < GV_STAGE; ++u) {
        const int i = i0 + u * nthr;
        v[u] = (i < n16 && i / KV < a.rows) ? src[i] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < GV_STAGE; ++u) {
        const int i = i0 + u * nthr, r = i / KV;
        if (i < n16) *reinterpret_cast<uint4*>(xs + (size_t)r * ld + (size_t)(i - r * KV) * VN) = v[u];
      }
    }
  } else {
    const int K4 = K / 4, n4 = ROWS * K4, nthr = nw * 32;
    const float4* src = reinterpret_cast<const float4*>(a.in);
    for (int i0 = threadIdx.x; i0 < n4; i0 += GV_STAGE * nthr) {
      float4 v[GV_STAGE];
#pragma unroll
      for (int u = 0; u < GV_STAGE; ++u) {
        const int i = i0 + u * nthr;
        v[u] = (i < n4 && i / K4 < a.rows) ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < GV_STAGE; ++u) {
        const int i = i0 + u * nthr;
        if (i < n4) {
          const int r = i / K4;
          T* d = xs + (size_t)r * ld + 4 * (i - r * K4);
          d[0] = from_f<T>(v[u].x);
          d[1] = from_f<T>(v[u].y);
          d[2] = from_f<T>(v[u].z);
          d[3] = from_f<T>(v[u].w);
        }
      }
    }
  }
}

// out[r, n] = epi(sum_k in'[r, k] W[n, k]) for r < rows, n < N, where in' is
// the input row (LN = true: its LayerNorm with eps 1e-5 and biased variance)
// rounded to T.  Each warp takes GV_COLS consecutive columns per pass; lane l
// reads 16-byte pieces l, l + 32, ... of each weight row.
// KS > 1 splits each column group's k-iterations over KS warps (iterations
// i = slice, slice + KS, ...); their totals meet in shared memory and the
// slice-0 warp applies the epilogue, summing the slices in a fixed order.
template <typename T, int ROWS, bool LN, int EPI, int KS>
__global__ void __launch_bounds__(GV_WARPS * 32) decode_gemv_kernel(const __grid_constant__ GemvArgs a) {
  extern __shared__ __align__(16) uint8_t dec_smem[];
  T* xs = reinterpret_cast<T*>(dec_smem);  // [ROWS][K]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;  // 4 or 8 warps
  const int K = a.K;
  constexpr int VN = V16<T>::N;
  constexpr int P = GV_COLS * ROWS;
  constexpr int HELD = P >= 32 ? P / 32 : 1;  // totals a lane holds after the reduction
  const T* W = reinterpret_cast<const T*>(a.W);
  const int groups = a.N / GV_COLS;
  const int gpc = nw / KS;                    // column groups per block and pass
  const int gi = warp / KS, si = warp % KS;   // this warp's group and k slice
  const int NI = (K + 32 * VN - 1) / (32 * VN);  // k-iterations of 32 x VN elements
  // (KS > 1) the slices' totals: [warp][HELD][lane], after the staged rows
  float* red = reinterpret_cast<float*>(dec_smem + (size_t)ROWS * K * sizeof(T));
  // GV_CHUNK of this slice's k-iterations of weight loads are issued together,
  // before the first FMA that uses them; the first chunk of a warp's next
  // column group is loaded ahead (here: before the input staging, whose
  // memory round trip it overlaps; later: before the reduction of the
  // previous group)
  uint4 wv[GV_CHUNK][GV_COLS];
  auto load_chunk = [&](int g, int it0) {
    const T* w0 = W + (size_t)g * GV_COLS * K;
#pragma unroll
    for (int u = 0; u < GV_CHUNK; ++u) {
      const int k = lane * VN + (it0 + u * KS) * 32 * VN;
#pragma unroll
      for (int c = 0; c < GV_COLS; ++c)
        wv[u][c] = k < K ? ld_stream16(w0 + (size_t)c * K + k) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // The first weight chunk is loaded before the grid-dependency wait: no
  // kernel of the decode step writes weights, and the step's first kernel
  // (the embedding) lets its successors start only after every kernel before
  // the step has finished.  The loads then overlap the predecessor's tail.
  pdl_trigger();
  if (blockIdx.x * gpc + gi < groups) load_chunk(blockIdx.x * gpc + gi, si);
  pdl_wait();

  gemv_stage_rows<T, ROWS, LN>(a, xs, K, warp, lane, nw);
  __syncthreads();

  // passes over the column groups, uniform across the block (the slices of a
  // group synchronise through shared memory once per pass)
  for (int pass_base = blockIdx.x * gpc; pass_base < groups; pass_base += gridDim.x * gpc) {
    const int grp = pass_base + gi;
    const bool active = grp < groups;
    const int n0 = grp * GV_COLS;
    // the epilogue's operands (bias, old residual, cache position) are loaded
    // now, so that their latency hides behind the weight stream
    float pre_b[HELD], pre_x[HELD];
    int pre_p[HELD];
#pragma unroll
    for (int j = 0; j < HELD; ++j) {
      bool owner;
      const int idx = rs_index<P>(lane, j, &owner);
      const int c = idx / ROWS, r = idx % ROWS;
      const bool live = active && si == 0 && owner && r < a.rows;
      pre_b[j] = 0.f;
      pre_x[j] = 0.f;
      pre_p[j] = 0;
      if (live) {
        if constexpr (EPI != DEC_LOGITS) pre_b[j] = to_f(reinterpret_cast<const T*>(a.bias)[n0 + c]);
        if constexpr (EPI == DEC_RESID) pre_x[j] = reinterpret_cast<const float*>(a.out)[(size_t)r * a.ldo + n0 + c];
        if constexpr (EPI == DEC_QKV) pre_p[j] = a.pos[r];
      }
    }
    float acc[P];
#pragma unroll
    for (int i = 0; i < P; ++i) acc[i] = 0.f;
    if (active) {
      for (int it0 = si; it0 < NI; it0 += GV_CHUNK * KS) {
        if (it0 != si) load_chunk(grp, it0);
#pragma unroll
        for (int u = 0; u < GV_CHUNK; ++u) {
          const int k = lane * VN + (it0 + u * KS) * 32 * VN;
          if (k >= K) break;
          float wf[GV_COLS][VN];
#pragma unroll
          for (int c = 0; c < GV_COLS; ++c) V16<T>::unpack(wv[u][c], wf[c]);
          // two rows per packed fp32x2 multiply-add (each lane of the pair
          // rounds like fmaf, in the same order: the sums are unchanged)
#pragma unroll
          for (int r = 0; r < ROWS; r += 2) {
            float xa[VN], xb[VN];
            V16<T>::unpack(*reinterpret_cast<const uint4*>(xs + (size_t)r * K + k), xa);
            V16<T>::unpack(*reinterpret_cast<const uint4*>(xs + (size_t)(r + 1) * K + k), xb);
#pragma unroll
            for (int c = 0; c < GV_COLS; ++c) {
              float2 a2 = make_float2(acc[c * ROWS + r], acc[c * ROWS + r + 1]);
#pragma unroll
              for (int e = 0; e < VN; ++e)
                a2 = __ffma2_rn(make_float2(wf[c][e], wf[c][e]), make_float2(xa[e], xb[e]), a2);
              acc[c * ROWS + r] = a2.x;
              acc[c * ROWS + r + 1] = a2.y;
            }
          }
        }
      }
      if (grp + (int)gridDim.x * gpc < groups) load_chunk(grp + gridDim.x * gpc, si);
    }
    ReduceScatter<P, 16>::run(acc, lane);
    if constexpr (KS > 1) {
#pragma unroll
      for (int j = 0; j < HELD; ++j) red[(warp * HELD + j) * 32 + lane] = acc[j];
      __syncthreads();
      if (si == 0) {
#pragma unroll
        for (int j = 0; j < HELD; ++j) {
          float t = acc[j];
#pragma unroll
          for (int x = 1; x < KS; ++x) t += red[((warp + x) * HELD + j) * 32 + lane];
          acc[j] = t;
        }
      }
    }
    if (active && si == 0) {
#pragma unroll
      for (int j = 0; j < HELD; ++j) {
        bool owner;
        const int idx = rs_index<P>(lane, j, &owner);
        const int c = idx / ROWS, r = idx % ROWS;
        if (!owner || r >= a.rows) continue;
        const int n = n0 + c;
        const float v = acc[j] + pre_b[j];
        float* outf = reinterpret_cast<float*>(a.out);
        if constexpr (EPI == DEC_QKV) {
          if (n < a.d) {
            outf[(size_t)r * a.ldo + n] = v;
          } else {
            const int kind = n >= 2 * a.d;
            const int nn = n - a.d - kind * a.d;
            const int p = pre_p[j];
            if (p >= 0 && p < a.max_len) {
              T* plane = reinterpret_cast<T*>(kind ? a.vc : a.kc);
              plane[(((size_t)r * a.H + nn / a.hd) * a.max_len + p) * a.hd + nn % a.hd] = from_f<T>(v);
            }
          }
        } else if constexpr (EPI == DEC_RESID) {
          outf[(size_t)r * a.ldo + n] = pre_x[j] + v;
        } else if constexpr (EPI == DEC_GELU) {
          reinterpret_cast<T*>(a.out)[(size_t)r * a.ldo + n] = from_f<T>(gelu_f<false>(v));
        } else {
          outf[(size_t)r * a.ldo + n] = v;
        }
      }
    }
    // the next pass overwrites red only after every slice-0 warp has read it
    if constexpr (KS > 1) __syncthreads();
  }
}

// ------------------------------------------------------ tensor-core GEMV --
// The same products for bf16 and at most 8 rows on mma.sync m16n8k16: the
// weights are the A operand (16 weight rows, i.e. 16 output columns, per
// warp), the staged rows the B operand (N 8; rows past a.rows are zero).  Per
// 32 k-elements a lane loads 16 bytes of each of its two weight rows (g and
// g + 8 of the warp's 16, g = lane / 4) and the 16 bytes of staged row g at
// the same k; within those 32 elements both operands take the same
// permutation of the fragment's k order (lane quad t holds elements 8t ..
// 8t + 7; the first mma reads 8t .. 8t + 3 of each, the second 8t + 4 ..
// 8t + 7), so the loads are the fragments as they stand.  Each (column, row)
// total ends on one lane, with no cross-lane reduction; KS warps split a
// group's k range and add their parts in shared memory in a fixed order.  At
// 8 rows a weight element feeds 8 products, so the dot products would
// otherwise cost as many CUDA-core instructions as the weight stream allows
// loads; on the tensor core they are a few instructions per 32 elements.
constexpr int MG_COLS = 16;  // output columns per warp (the mma M)
constexpr int MG_KC = 32;    // k elements per lane load of a weight row
constexpr int MG_U = 4;      // k chunks of weight loads in flight per batch
constexpr int MG_PAD = 32;   // elements (64 bytes) after each staged row: the 8
                             // rows' 16-byte fragment loads then avoid bank conflicts

DEVI void gemv_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool LN, int EPI, int KS>
__global__ void __launch_bounds__(GV_WARPS * 32) decode_gemv_mma_kernel(const __grid_constant__ GemvArgs a) {
  extern __shared__ __align__(16) uint8_t dec_smem[];
  constexpr int GPB = GV_WARPS / KS;  // column groups per block and pass
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int K = a.K, ld = K + MG_PAD;
  bf16* xs = reinterpret_cast<bf16*>(dec_smem);                              // [8][ld]
  float* red = reinterpret_cast<float*>(dec_smem + (size_t)8 * ld * sizeof(bf16));  // [warps][32][4]
  const bf16* W = reinterpret_cast<const bf16*>(a.W);
  const int groups = a.N / MG_COLS;
  const int gi = warp / KS, si = warp % KS;
  const int nch = K / MG_KC;
  const int c0 = si * nch / KS, c1 = (si + 1) * nch / KS;  // this warp's k chunks
  const int nb = (c1 - c0 + MG_U - 1) / MG_U;              // batches of them per group
  uint4 wa[MG_U], wb[MG_U], na[MG_U], nb_[MG_U];
  // batch b of group grp: chunks c0 + MG_U b + u < c1, rows g and g + 8
  auto load_batch = [&](uint4 (&x0)[MG_U], uint4 (&x1)[MG_U], int grp, int b) {
    const bf16* w0 = W + (size_t)(grp * MG_COLS + g) * K + 8 * t;
    const bf16* w1 = w0 + (size_t)8 * K;
#pragma unroll
    for (int u = 0; u < MG_U; ++u) {
      const int ch = c0 + b * MG_U + u;
      if (ch < c1) {
        x0[u] = ld_stream16(w0 + ch * MG_KC);
        x1[u] = ld_stream16(w1 + ch * MG_KC);
      }
    }
  };
  // The first batch is requested before the grid-dependency wait, as in
  // decode_gemv_kernel (no kernel of the decode step writes weights).
  pdl_trigger();
  if (blockIdx.x * GPB + gi < groups && nb > 0) load_batch(wa, wb, blockIdx.x * GPB + gi, 0);
  pdl_wait();
  gemv_stage_rows<bf16, 8, LN>(a, xs, ld, warp, lane, GV_WARPS);
  __syncthreads();

  for (int pass_base = blockIdx.x * GPB; pass_base < groups; pass_base += gridDim.x * GPB) {
    const int grp = pass_base + gi;
    const bool active = grp < groups;
    const int n0 = grp * MG_COLS;
    // the epilogue's operands (bias, old residual, cache positions) of this
    // lane's outputs (columns n0 + g, n0 + g + 8; rows 2t, 2t + 1), loaded
    // now so that their latency hides behind the products
    float pre_b[2] = {0.f, 0.f}, pre_x[4] = {0.f, 0.f, 0.f, 0.f};
    int pre_p[2] = {0, 0};
    if (active && si == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + g + 8 * h;
        if constexpr (EPI != DEC_LOGITS) pre_b[h] = to_f(reinterpret_cast<const bf16*>(a.bias)[n]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int r = 2 * t + j;
          if constexpr (EPI == DEC_RESID)
            if (r < a.rows) pre_x[2 * h + j] = reinterpret_cast<const float*>(a.out)[(size_t)r * a.ldo + n];
        }
      }
      if constexpr (EPI == DEC_QKV) {
#pragma unroll
        for (int j = 0; j < 2; ++j) pre_p[j] = 2 * t + j < a.rows ? a.pos[2 * t + j] : 0;
      }
    }
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    if (active) {
      for (int b = 0; b < nb; ++b) {
        // the next batch (of this group, else the first of this warp's next
        // group) is requested before this one is used
        const int ngrp = grp + (int)gridDim.x * GPB;
        if (b + 1 < nb)
          load_batch(na, nb_, grp, b + 1);
        else if (ngrp < groups)
          load_batch(na, nb_, ngrp, 0);
#pragma unroll
        for (int u = 0; u < MG_U; ++u) {
          const int ch = c0 + b * MG_U + u;
          if (ch < c1) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)g * ld + ch * MG_KC + 8 * t);
            gemv_mma(c, wa[u].x, wb[u].x, wa[u].y, wb[u].y, xv.x, xv.y);
            gemv_mma(c, wa[u].z, wb[u].z, wa[u].w, wb[u].w, xv.z, xv.w);
          }
        }
#pragma unroll
        for (int u = 0; u < MG_U; ++u) {
          wa[u] = na[u];
          wb[u] = nb_[u];
        }
      }
    }
    if constexpr (KS > 1) {
      *reinterpret_cast<float4*>(red + (warp * 32 + lane) * 4) = make_float4(c[0], c[1], c[2], c[3]);
      __syncthreads();
      if (si == 0) {
#pragma unroll
        for (int x = 1; x < KS; ++x) {
          const float4 q = *reinterpret_cast<const float4*>(red + ((warp + x) * 32 + lane) * 4);
          c[0] += q.x;
          c[1] += q.y;
          c[2] += q.z;
          c[3] += q.w;
        }
      }
    }
    if (active && si == 0) {
      // c[i]: column n0 + g + 8 (i / 2), row 2t + i % 2
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int h = i >> 1, r = 2 * t + (i & 1);
        if (r >= a.rows) continue;
        const int n = n0 + g + 8 * h;
        const float v = c[i] + pre_b[h];
        float* outf = reinterpret_cast<float*>(a.out);
        if constexpr (EPI == DEC_QKV) {
          if (n < a.d) {
            outf[(size_t)r * a.ldo + n] = v;
          } else {
            const int kind = n >= 2 * a.d;
            const int nn = n - a.d - kind * a.d;
            const int p = pre_p[i & 1];
            if (p >= 0 && p < a.max_len) {
              bf16* plane = reinterpret_cast<bf16*>(kind ? a.vc : a.kc);
              plane[(((size_t)r * a.H + nn / a.hd) * a.max_len + p) * a.hd + nn % a.hd] = from_f<bf16>(v);
            }
          }
        } else if constexpr (EPI == DEC_RESID) {
          outf[(size_t)r * a.ldo + n] = pre_x[i] + v;
        } else if constexpr (EPI == DEC_GELU) {
          reinterpret_cast<bf16*>(a.out)[(size_t)r * a.ldo + n] = from_f<bf16>(gelu_f<false>(v));
        } else {
          outf[(size_t)r * a.ldo + n] = c[i];
        }
      }
    }
    // the next pass overwrites red only after every slice-0 warp has read it
    if constexpr (KS > 1) __syncthreads();
  }
}

// x[r, :] = wte[tok[r]] + wpe[pos[r]] (fp32); an id outside [0, vocab_real)
// or a position outside [0, limit) raises its status bit and reads row 0.
template <typename T>
__global__ void embed_decode_kernel(const int32_t* tok, const int32_t* pos,
                                    const T* wte, const T* wpe, float* __restrict__ x,
                                    int d, int vocab_real, int limit, int* err) {
  // wait before letting the step's kernels start: they load weights before
  // their own waits, and a kernel before the step may still be writing them
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  int id = tok[r], p = pos[r];
  if (id < 0 || id >= vocab_real) {
    if (threadIdx.x == 0) atomicOr(err, DEV_ERR_TOKEN);
    id = 0;
  }
  if (p < 0 || p >= limit) {
    if (threadIdx.x == 0) atomicOr(err, DEV_ERR_POSITION);
    p = 0;
  }
  for (int k = threadIdx.x; k < d; k += blockDim.x)
    x[(size_t)r * d + k] = to_f(wte[(size_t)id * d + k]) + to_f(wpe[(size_t)p * d + k]);
}

constexpr int AD_WARPS = 8;

// Attention of row r's new query (head h) against its cached positions
// 0..pos[r]: each warp takes 32-position tiles t = warp, warp + 8, ...; lane
// j of a tile loads key and value row 32 t + j with 16-byte loads, scores the
// key, and keeps its own weighted sum of values relative to the warp's running
// maximum, so a tile costs two memory round trips and no per-position
// shuffles.  At the end the lanes' sums are reduced within the warp and the
// warps' results merged through shared memory.
template <typename T, int HD>
__global__ void __launch_bounds__(AD_WARPS * 32)
    attn_decode_kernel(const T* kc, const T* vc, const float* q,
                       float* __restrict__ o, const int32_t* pos, int H, int max_len,
                       float scale_log2) {
  __shared__ float sm_m[AD_WARPS], sm_l[AD_WARPS];
  __shared__ float sm_o[AD_WARPS][HD];
  pdl_trigger();
  const int h = blockIdx.x, r = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = H * HD;
  // positions come from before the step (the step's first kernel waited for
  // their writers), and so do the cached rows of positions < p: the warp's
  // first tile of those is loaded ahead of the grid-dependency wait; row p
  // (written by the QKV product just before) and q only after it
  int p = pos[r];
  p = p < 0 ? 0 : (p >= max_len ? max_len - 1 : p);  // out of range: flagged by the embedding
  const int n = p + 1;
  constexpr int VN = V16<T>::N;
  const size_t plane = ((size_t)r * H + h) * max_len * HD;
  const T* kb = kc + plane;
  const T* vb = vc + plane;
  // (bf16 rows: the fp32 rows of the correctness mode do not fit twice in registers)
  constexpr bool PRE = sizeof(T) == 2;
  const int j0 = warp * 32 + lane;
  const bool early = PRE && j0 < p;
  uint4 kr0[HD / VN], vr0[HD / VN];
  if (early) {
#pragma unroll
    for (int c = 0; c < HD / VN; ++c) kr0[c] = *reinterpret_cast<const uint4*>(kb + (size_t)j0 * HD + c * VN);
#pragma unroll
    for (int c = 0; c < HD / VN; ++c) vr0[c] = *reinterpret_cast<const uint4*>(vb + (size_t)j0 * HD + c * VN);
  }
  pdl_wait();
  float qf[HD];
#pragma unroll
  for (int i = 0; i < HD; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(q + (size_t)r * d + h * HD + i);
    qf[i] = v.x * scale_log2; qf[i + 1] = v.y * scale_log2; qf[i + 2] = v.z * scale_log2; qf[i + 3] = v.w * scale_log2;
  }
  float m = -INFINITY, l = 0.f, acc[HD];
#pragma unroll
  for (int e = 0; e < HD; ++e) acc[e] = 0.f;
  for (int t = warp; t * 32 < n; t += AD_WARPS) {
    const int j = t * 32 + lane;
    const int jr = j < n ? j : n - 1;  // rows past n are read in bounds and weighted 0
    uint4 kr[HD / VN], vr[HD / VN];
    if (t == warp && early) {
#pragma unroll
      for (int c = 0; c < HD / VN; ++c) {
        kr[c] = kr0[c];
        vr[c] = vr0[c];
      }
    } else {
#pragma unroll
      for (int c = 0; c < HD / VN; ++c) kr[c] = *reinterpret_cast<const uint4*>(kb + (size_t)jr * HD + c * VN);
      if constexpr (PRE) {
#pragma unroll
        for (int c = 0; c < HD / VN; ++c) vr[c] = *reinterpret_cast<const uint4*>(vb + (size_t)jr * HD + c * VN);
      }
    }
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < HD / VN; ++c) {
      float kf[VN];
      V16<T>::unpack(kr[c], kf);
#pragma unroll
      for (int e = 0; e < VN; ++e) s = fmaf(qf[c * VN + e], kf[e], s);
    }
    if (j >= n) s = -INFINITY;
    const float mnew = fmaxf(m, warp_max(s));  // lane 0's key is always valid
    const float alpha = ex2_approx(m - mnew);
    const float pj = ex2_approx(s - mnew);
    m = mnew;
    l = l * alpha + pj;
#pragma unroll
    for (int c = 0; c < HD / VN; ++c) {
      float vf[VN];
      V16<T>::unpack(PRE ? vr[c] : *reinterpret_cast<const uint4*>(vb + (size_t)jr * HD + c * VN), vf);
#pragma unroll
      for (int e = 0; e < VN; ++e) acc[c * VN + e] = fmaf(pj, vf[e], acc[c * VN + e] * alpha);
    }
  }
  l = warp_sum(l);
  ReduceScatter<HD, 16>::run(acc, lane);
  constexpr int HELD = HD >= 32 ? HD / 32 : 1;
#pragma unroll
  for (int jj = 0; jj < HELD; ++jj) {
    bool owner;
    const int idx = rs_index<HD>(lane, jj, &owner);
    if (owner) sm_o[warp][idx] = acc[jj];
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_l[warp] = l;
  }
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < AD_WARPS; ++w) M = fmaxf(M, sm_m[w]);
    float L = 0.f;
    float f[AD_WARPS];
#pragma unroll
    for (int w = 0; w < AD_WARPS; ++w) {
      f[w] = sm_m[w] == -INFINITY ? 0.f : ex2_approx(sm_m[w] - M);  // a warp with no tile weighs 0
      L += sm_l[w] * f[w];
    }
    const float inv = 1.f / L;
    for (int e = lane; e < HD; e += 32) {
      float out = 0.f;
#pragma unroll
      for (int w = 0; w < AD_WARPS; ++w) out += sm_o[w][e] * f[w];
      o[(size_t)r * d + h * HD + e] = out * inv;
    }
  }
}

// (value, id) order of the greedy choice: NaN above everything, then larger
// values, then the lower id.
DEVI bool greedy_better(float a, int ia, float b, int ib) {
  const bool na = a != a, nb = b != b;
  if (na != nb) return na;
  if (!na && a != b) return a > b;
  return ia < ib;
}

// next[r] = argmax over v < vocab_real of logits[r, v]; pos[r] += 1 if pos.
__global__ void __launch_bounds__(1024)
    greedy_kernel(const float* logits, long ld, int vocab_real, int32_t* __restrict__ next,
                  int32_t* __restrict__ pos) {
  __shared__ float sv[32];
  __shared__ int si[32];
  pdl_start();
  const int r = blockIdx.x;
  const float* z = logits + (size_t)r * ld;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  constexpr int U = 8;  // loads in flight per thread
  for (int v0 = threadIdx.x; v0 < vocab_real; v0 += U * blockDim.x) {
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * blockDim.x;
      x[u] = v < vocab_real ? z[v] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * blockDim.x;
      if (v < vocab_real && greedy_better(x[u], v, bv, bi)) {
        bv = x[u];
        bi = v;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (greedy_better(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sv[warp] = bv;
    si[warp] = bi;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    bv = lane < nw ? sv[lane] : -INFINITY;
    bi = lane < nw ? si[lane] : 0x7fffffff;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (greedy_better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      next[r] = bi < vocab_real ? bi : 0;
      if (pos) pos[r] += 1;
    }
  }
}

// The greedy choice over many blocks (rows <= GREEDY_SPLIT_MAX_ROWS): block
// (s, r) scans slice s of row r's real vocabulary and leaves its best
// (value, id); one warp per row then picks the best of the GREEDY_SLICES.
constexpr int GREEDY_SLICES = 16;
__global__ void __launch_bounds__(256)
    greedy_part_kernel(const float* logits, long ld, int vocab_real, float* __restrict__ pv,
                       int* __restrict__ pi) {
  __shared__ float sv[8];
  __shared__ int si[8];
  pdl_start();
  const int s = blockIdx.x, r = blockIdx.y;
  const int per = (vocab_real + GREEDY_SLICES - 1) / GREEDY_SLICES;
  const int v0 = s * per, v1 = min(vocab_real, v0 + per);
  const float* z = logits + (size_t)r * ld;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  constexpr int U = 8;
  for (int b0 = v0 + (int)threadIdx.x; b0 < v1; b0 += U * 256) {
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) x[u] = b0 + u * 256 < v1 ? z[b0 + u * 256] : -INFINITY;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = b0 + u * 256;
      if (v < v1 && greedy_better(x[u], v, bv, bi)) {
        bv = x[u];
        bi = v;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (greedy_better(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sv[warp] = bv;
    si[warp] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w)
      if (greedy_better(sv[w], si[w], bv, bi)) {
        bv = sv[w];
        bi = si[w];
      }
    pv[r * GREEDY_SLICES + s] = bv;
    pi[r * GREEDY_SLICES + s] = bi;
  }
}

__global__ void greedy_final_kernel(const float* pv, const int* pi, int vocab_real,
                                    int32_t* __restrict__ next, int32_t* __restrict__ pos) {
  pdl_start();
  const int r = blockIdx.x, lane = threadIdx.x;
  float bv = lane < GREEDY_SLICES ? pv[r * GREEDY_SLICES + lane] : -INFINITY;
  int bi = lane < GREEDY_SLICES ? pi[r * GREEDY_SLICES + lane] : 0x7fffffff;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (greedy_better(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  if (lane == 0) {
    next[r] = bi < vocab_real ? bi : 0;
    if (pos) pos[r] += 1;
  }
}

// Prefill: K and V of positions < plen[r] from a layer's qkv activation
// [rows * T, 3d] into the cache planes; plen outside [1, limit] raises the
// position bit and copies nothing for that row.
template <typename T>
__global__ void prefill_kv_kernel(const T* qkv, T* __restrict__ kc, T* __restrict__ vc,
                                  const int32_t* plen, int T_ctx, int H, int hd, int max_len,
                                  int limit, int* err) {
  pdl_start();
  const int p = blockIdx.x, r = blockIdx.y;
  const int n = plen[r];
  if (n < 1 || n > limit) {
    if (p == 0 && threadIdx.x == 0 && err) atomicOr(err, DEV_ERR_POSITION);
    return;
  }
  if (p >= n) return;
  const int d = H * hd;
  const T* src = qkv + ((size_t)r * T_ctx + p) * 3 * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const size_t dst = (((size_t)r * H + c / hd) * max_len + p) * hd + c % hd;
    kc[dst] = src[d + c];
    vc[dst] = src[2 * d + c];
  }
}

// logits_out[r, :] = logits[r * T + plen[r] - 1, :] in fp32 (plen clamped to
// [1, limit]; the position bit is raised by the K/V copy).
template <typename T>
__global__ void prefill_logits_kernel(const T* logits, const int32_t* plen,
                                      float* __restrict__ out, int T_ctx, int V, int limit) {
  pdl_start();
  const int r = blockIdx.y;
  int n = plen[r];
  n = n < 1 ? 1 : (n > limit ? limit : n);
  const T* src = logits + ((size_t)r * T_ctx + n - 1) * V;
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < V; v += gridDim.x * blockDim.x)
    out[(size_t)r * V + v] = to_f(src[v]);
}

template <typename T, int ROWS, bool LN, int EPI, int KS>
int gemv_launch(const GemvArgs& a, cudaStream_t st) {
  constexpr int HELD = GV_COLS * ROWS >= 32 ? GV_COLS * ROWS / 32 : 1;
  const size_t smem = (size_t)ROWS * a.K * sizeof(T) + (KS > 1 ? (size_t)GV_WARPS * HELD * 32 * 4 : 0);
  CUDA_TRY(once_per_device((const void*)decode_gemv_kernel<T, ROWS, LN, EPI, KS>, [](int) {
    return cudaFuncSetAttribute(decode_gemv_kernel<T, ROWS, LN, EPI, KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                227 * 1024);
  }));
  const int groups = a.N / GV_COLS;
  // narrow outputs: 4-warp blocks (or, with a k split, 8 warps on 2 groups),
  // so that more SMs stream weights
  const int nw = (KS > 1 || LN || groups >= GV_WARPS * num_sms()) ? GV_WARPS : 4;
  const int gpc = nw / KS;
  int grid = (groups + gpc - 1) / gpc;
  // at most one wave of resident blocks (the registers allow one 8-warp block
  // per SM): a second wave would repeat the input staging and add a tail
  static int per_sm[MAX_DEVICES][2] = {};
  int& occ = per_sm[current_device()][nw == GV_WARPS];
  if (occ == 0 && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_gemv_kernel<T, ROWS, LN, EPI, KS>,
                                                                   nw * 32, smem) != cudaSuccess || occ < 1))
    occ = 1;
  const int cap = occ * num_sms();
  if (grid > cap) grid = cap;
  CUDA_TRY(launch_k(decode_gemv_kernel<T, ROWS, LN, EPI, KS>, grid, nw * 32, smem, st, a));
  LAUNCH_CHECK();
  return GPT2_OK;
}

template <typename T, bool LN, int EPI, int KS>
int gemv_rows(const GemvArgs& a, cudaStream_t st) {
  if (a.rows <= 4) return gemv_launch<T, 4, LN, EPI, KS>(a, st);
  if (a.rows <= 8) return gemv_launch<T, 8, LN, EPI, KS>(a, st);
  return gemv_launch<T, 16, LN, EPI, KS>(a, st);
}

template <bool LN, int EPI, int KS>
int gemv_mma_launch(const GemvArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)8 * (a.K + MG_PAD) * sizeof(bf16) + (size_t)GV_WARPS * 32 * 16;
  CUDA_TRY(once_per_device((const void*)decode_gemv_mma_kernel<LN, EPI, KS>, [](int) {
    return cudaFuncSetAttribute(decode_gemv_mma_kernel<LN, EPI, KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                227 * 1024);
  }));
  constexpr int GPB = GV_WARPS / KS;
  const int groups = a.N / MG_COLS;
  int grid = (groups + GPB - 1) / GPB;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_gemv_mma_kernel<LN, EPI, KS>, GV_WARPS * 32, smem) !=
          cudaSuccess || occ < 1)
    occ = 1;
  if (grid > occ * num_sms()) grid = occ * num_sms();  // one resident wave
  CUDA_TRY(launch_k(decode_gemv_mma_kernel<LN, EPI, KS>, grid, GV_WARPS * 32, smem, st, a));
  LAUNCH_CHECK();
  return GPT2_OK;
}

// the k split: all 8 warps of a block on one 16-column group while the
// groups fit one block per SM, fewer as they grow
template <bool LN, int EPI>
int gemv_mma_ks(const GemvArgs& a, cudaStream_t st) {
  const int groups = a.N / MG_COLS;
  if (groups <= num_sms()) return gemv_mma_launch<LN, EPI, 8>(a, st);
  if (groups <= 2 * num_sms()) return gemv_mma_launch<LN, EPI, 4>(a, st);
  return gemv_mma_launch<LN, EPI, 2>(a, st);
}

template <typename T>
int gemv_dispatch(const GemvArgs& a, bool ln, int epi, cudaStream_t st) {
  // the residual products have narrow outputs (d columns): k split four ways
  // (for the LayerNorm'd products a split measured slower: every extra block
  // repeats the LayerNorm of the staged rows)
  if (epi == DEC_QKV && ln) return gemv_rows<T, true, DEC_QKV, 1>(a, st);
  if (epi == DEC_RESID && !ln) return gemv_rows<T, false, DEC_RESID, 4>(a, st);
  if (epi == DEC_GELU && ln) return gemv_rows<T, true, DEC_GELU, 1>(a, st);
  if (epi == DEC_LOGITS && ln) return gemv_rows<T, true, DEC_LOGITS, 1>(a, st);
  return GPT2_ERR_INVALID_ARG;
}

}  // namespace

size_t decode_gemv_smem(int f32, int rows, int K) {
  const int R = rows <= 4 ? 4 : (rows <= 8 ? 8 : 16);
  return (size_t)R * K * (f32 ? 4 : 2) + (size_t)GV_WARPS * (R / 8 > 1 ? R / 8 : 1) * 32 * 4;
}

int decode_embed(int f32, const int32_t* tok, const int32_t* pos, const void* wte, const void* wpe, float* x,
                 int rows, int d, int vocab_real, int limit, int* err, cudaStream_t st) {
  if (f32)
    CUDA_TRY(launch_k(embed_decode_kernel<float>, rows, 256, 0, st, tok, pos, (const float*)wte,
                      (const float*)wpe, x, d, vocab_real, limit, err));
  else
    CUDA_TRY(launch_k(embed_decode_kernel<bf16>, rows, 256, 0, st, tok, pos, (const bf16*)wte, (const bf16*)wpe,
                      x, d, vocab_real, limit, err));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int decode_gemv(int f32, const DecodeGemv& g, cudaStream_t st) {
  if (g.N % GV_COLS || g.K % 64 || g.rows < 1 || g.rows > 16) return GPT2_ERR_INVALID_ARG;
  if (g.ln && g.K > LN_MAX_K) return GPT2_ERR_UNSUPPORTED_SHAPE;
  GemvArgs a;
  a.in = g.in; a.in_t = g.in_t; a.W = g.W; a.bias = g.bias; a.ln_g = g.ln_g; a.ln_b = g.ln_b;
  a.out = g.out; a.ldo = g.ldo; a.rows = g.rows; a.N = g.N; a.K = g.K;
  a.kc = g.kc; a.vc = g.vc; a.pos = g.pos; a.d = g.d; a.H = g.H; a.hd = g.hd; a.max_len = g.max_len;
  // bf16 at up to 8 rows: the tensor-core GEMV ("simt" in GPT2_DECODE_GEMV
  // selects the CUDA-core kernel, for comparison)
  const char* e = getenv("GPT2_DECODE_GEMV");
  if (!f32 && g.rows <= 8 && g.N % MG_COLS == 0 && !(e && !strcmp(e, "simt"))) {
    if (g.epi == DEC_QKV && g.ln) return gemv_mma_ks<true, DEC_QKV>(a, st);
    if (g.epi == DEC_RESID && !g.ln) return gemv_mma_ks<false, DEC_RESID>(a, st);
    if (g.epi == DEC_GELU && g.ln) return gemv_mma_ks<true, DEC_GELU>(a, st);
    if (g.epi == DEC_LOGITS && g.ln) return gemv_mma_ks<true, DEC_LOGITS>(a, st);
    return GPT2_ERR_INVALID_ARG;
  }
  return f32 ? gemv_dispatch<float>(a, g.ln, g.epi, st) : gemv_dispatch<bf16>(a, g.ln, g.epi, st);
}

int decode_attention(int f32, const void* kc, const void* vc, const float* q, float* o, const int32_t* pos,
                     int rows, int H, int hd, int max_len, cudaStream_t st) {
  const dim3 grid(H, rows);
  const float sl2 = 1.4426950408889634f / sqrtf((float)hd);
  if (hd == 64) {
    if (f32)
      CUDA_TRY(launch_k(attn_decode_kernel<float, 64>, grid, AD_WARPS * 32, 0, st, (const float*)kc,
                        (const float*)vc, q, o, pos, H, max_len, sl2));
    else
      CUDA_TRY(launch_k(attn_decode_kernel<bf16, 64>, grid, AD_WARPS * 32, 0, st, (const bf16*)kc, (const bf16*)vc,
                        q, o, pos, H, max_len, sl2));
  } else if (hd == 16) {
    if (f32)
      CUDA_TRY(launch_k(attn_decode_kernel<float, 16>, grid, AD_WARPS * 32, 0, st, (const float*)kc,
                        (const float*)vc, q, o, pos, H, max_len, sl2));
    else
      CUDA_TRY(launch_k(attn_decode_kernel<bf16, 16>, grid, AD_WARPS * 32, 0, st, (const bf16*)kc, (const bf16*)vc,
                        q, o, pos, H, max_len, sl2));
  } else {
    return GPT2_ERR_UNSUPPORTED_SHAPE;
  }
  LAUNCH_CHECK();
  return GPT2_OK;
}

int decode_greedy(const float* logits, long ld, int rows, int vocab_real, int32_t* next, int32_t* pos,
                  float* part_v, int* part_i, cudaStream_t st) {
  if (part_v && part_i && rows <= GREEDY_SPLIT_MAX_ROWS) {
    CUDA_TRY(launch_k(greedy_part_kernel, dim3(GREEDY_SLICES, rows), 256, 0, st, logits, ld, vocab_real, part_v,
                      part_i));
    LAUNCH_CHECK();
    CUDA_TRY(launch_k(greedy_final_kernel, rows, 32, 0, st, (const float*)part_v, (const int*)part_i, vocab_real,
                      next, pos));
  } else {
    CUDA_TRY(launch_k(greedy_kernel, rows, 1024, 0, st, logits, ld, vocab_real, next, pos));
  }
  LAUNCH_CHECK();
  return GPT2_OK;
}

int prefill_kv(int f32, const void* qkv, void* kc, void* vc, const int32_t* plen, int rows, int T, int H, int hd,
               int max_len, int limit, int* err, cudaStream_t st) {
  const dim3 grid(limit, rows);
  if (f32)
    CUDA_TRY(launch_k(prefill_kv_kernel<float>, grid, 256, 0, st, (const float*)qkv, (float*)kc, (float*)vc, plen,
                      T, H, hd, max_len, limit, err));
  else
    CUDA_TRY(launch_k(prefill_kv_kernel<bf16>, grid, 256, 0, st, (const bf16*)qkv, (bf16*)kc, (bf16*)vc, plen, T,
                      H, hd, max_len, limit, err));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int prefill_logits(int f32, const void* logits, const int32_t* plen, float* out, int rows, int T, int V, int limit,
                   cudaStream_t st) {
  const dim3 grid((V + 1023) / 1024, rows);
  if (f32)
    CUDA_TRY(launch_k(prefill_logits_kernel<float>, grid, 1024, 0, st, (const float*)logits, plen, out, T, V,
                      limit));
  else
    CUDA_TRY(launch_k(prefill_logits_kernel<bf16>, grid, 1024, 0, st, (const bf16*)logits, plen, out, T, V,
                      limit));
  LAUNCH_CHECK();
  return GPT2_OK;
}
