// Causal multi-head self-attention, forward and backward, softmax(q k^T /
// sqrt(hd), keys j <= query i) v per (batch, head).  "Pré-treinar um LLM"
// (Kaplan Eq. (2.2) paragraph) names this O(T^2) score term as the part of the
// step that 6ND leaves out.  The T x T scores never leave the chip: the
// forward keeps a running max / sum per query row (online softmax) and stores
// only O and the per-row log-sum-exp; the backward recomputes P tile by tile
// from q, k and that log-sum-exp.
//
// bf16 path: warp-level mma.sync m16n8k16 tiles (fp32 accumulation), cp.async
// double-buffered K/V (forward) and Q/dO (backward) tiles in XOR-swizzled
// shared memory, ldmatrix fragment loads.  Backward: one CTA per 64-key block
// accumulates dK, dV in registers over the query blocks at or below the
// diagonal; dQ contributions go to an fp32 buffer with vector reductions.
// fp32 path (correctness mode): plain CUDA-core kernels.
#include <stdlib.h>

#include "common.cuh"
#include "internal.h"

namespace {

#define LOG2E_F 1.4426950408889634f
#define LN2_F 0.6931471805599453f

DEVI void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
DEVI void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
DEVI void ldsm4t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
DEVI void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
DEVI void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
DEVI void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
DEVI void red_add_v2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

// Byte offset of 16-byte chunk c of row r in a tile whose rows hold NC chunks,
// with the chunk index XOR-swizzled by the row so ldmatrix is conflict-free.
template <int NC>
DEVI uint32_t swz(int r, int c) {
  return (uint32_t)(r * NC * 16 + ((c ^ (r & (NC - 1))) << 4));
}

// ----------------------------------------------------------------- forward --

template <int HD>
__global__ void __launch_bounds__(256) attn_fwd_kernel(const bf16* qkv,
                                                       bf16* __restrict__ o, float* __restrict__ lse,
                                                       int T, int H, float scale_log2) {
  pdl_start();
  constexpr int BQ = 128, BKV = 64, NC = HD / 8;
  constexpr int TILE_KV = BKV * HD * 2;
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sQ = smem_u32(sm);
  const uint32_t sK = sQ + BQ * HD * 2;
  const uint32_t sV = sK + 2 * TILE_KV;

  const int nqb = (T + BQ - 1) / BQ;
  const int qb = nqb - 1 - blockIdx.x;  // longest (causal) blocks first
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int d = H * HD;
  const long ld = 3L * d;
  const bf16* Qg = qkv + (long)b * T * ld + h * HD;
  const bf16* Kg = Qg + d;
  const bf16* Vg = Qg + 2 * d;
  const int q0 = qb * BQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < BQ * NC; i += 256) {
    int r = i / NC, c = i % NC, t = q0 + r;
    cp_async16(sQ + swz<NC>(r, c), Qg + (long)min(t, T - 1) * ld + c * 8, t < T ? 16 : 0);
  }
  cp_commit();
  auto load_kv = [&](int j, int buf) {
    for (int i = threadIdx.x; i < BKV * NC; i += 256) {
      int r = i / NC, c = i % NC, t = j * BKV + r;
      long off = (long)min(t, T - 1) * ld + c * 8;
      int bytes = t < T ? 16 : 0;
      cp_async16(sK + buf * TILE_KV + swz<NC>(r, c), Kg + off, bytes);
      cp_async16(sV + buf * TILE_KV + swz<NC>(r, c), Vg + off, bytes);
    }
  };
  const int q_last = min(q0 + BQ, T) - 1;
  const int nkv = q_last / BKV + 1;
  load_kv(0, 0);
  cp_commit();
  cp_wait<1>();
  __syncthreads();

  uint32_t qf[HD / 16][4];
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks) ldsm4(qf[ks], sQ + swz<NC>(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)));

  float oacc[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int r_lo = q0 + warp * 16 + (lane >> 2);
  const int warp_row0 = q0 + warp * 16;

  for (int j = 0; j < nkv; ++j) {
    if (j + 1 < nkv) load_kv(j + 1, (j + 1) & 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t kb = sK + (j & 1) * TILE_KV, vb = sV + (j & 1) * TILE_KV;
    const int kv0 = j * BKV;
    if (kv0 <= warp_row0 + 15) {  // else every key of this tile is in this warp's future
      float s[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          uint32_t kf[4];
          ldsm4(kf, kb + swz<NC>(n2 * 16 + (lane & 7) + ((lane >> 4) << 3), ks * 2 + ((lane >> 3) & 1)));
          mma16816(s[2 * n2], qf[ks], kf[0], kf[1]);
          mma16816(s[2 * n2 + 1], qf[ks], kf[2], kf[3]);
        }
      }
      const bool need_mask = (kv0 + BKV - 1 > warp_row0) || (kv0 + BKV > T);
      float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = s[n][e] * scale_log2;
          if (need_mask) {
            int col = kv0 + n * 8 + (lane & 3) * 2 + (e & 1);
            int row = r_lo + (e >> 1) * 8;
            if (col > row || col >= T) v = -INFINITY;
          }
          s[n][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
        mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      }
      float alpha[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        alpha[i] = exp2f(mrow[i] - mx[i]);
        mrow[i] = mx[i];
        lrow[i] *= alpha[i];
      }
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float p = exp2f(s[n][e] - mx[e >> 1]);
          s[n][e] = p;
          lrow[e >> 1] += p;
        }
      }
#pragma unroll
      for (int n = 0; n < HD / 8; ++n) {
        oacc[n][0] *= alpha[0]; oacc[n][1] *= alpha[0];
        oacc[n][2] *= alpha[1]; oacc[n][3] *= alpha[1];
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4] = {pack_bf16x2(s[2 * kk][0], s[2 * kk][1]), pack_bf16x2(s[2 * kk][2], s[2 * kk][3]),
                          pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                          pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3])};
#pragma unroll
        for (int n2 = 0; n2 < HD / 16; ++n2) {
          uint32_t vf[4];
          ldsm4t(vf, vb + swz<NC>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), n2 * 2 + (lane >> 4)));
          mma16816(oacc[2 * n2], pa, vf[0], vf[1]);
          mma16816(oacc[2 * n2 + 1], pa, vf[2], vf[3]);
        }
      }
    }
    __syncthreads();
  }

  float inv[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float l = lrow[i];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    lrow[i] = l;
    inv[i] = 1.f / l;
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int t = r_lo + hh * 8;
    if (t < T) {
      bf16* orow = o + ((long)b * T + t) * d + h * HD + (lane & 3) * 2;
#pragma unroll
      for (int n = 0; n < HD / 8; ++n)
        *reinterpret_cast<uint32_t*>(orow + n * 8) =
            pack_bf16x2(oacc[n][2 * hh] * inv[hh], oacc[n][2 * hh + 1] * inv[hh]);
      if ((lane & 3) == 0) lse[((long)b * H + h) * T + t] = (mrow[hh] + log2f(lrow[hh])) * LN2_F;
    }
  }
}

// ---------------------------------------------------------------- backward --

// D[b,h,t] = sum_c dO[t,c] O[t,c]; also zeroes the fp32 dQ accumulator.
template <typename T_>
__global__ void attn_bwd_prep_kernel(const T_* o, const T_* dout,
                                     float* __restrict__ dvec, float* __restrict__ dq_acc, int B,
                                     int T, int H, int hd) {
  pdl_start();
  long idx = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (idx >= (long)B * T * H) return;
  const int h = idx % H;
  const long m = idx / H;
  const int d = H * hd;
  const T_* op = o + m * d + h * hd;
  const T_* dp = dout + m * d + h * hd;
  float acc = 0.f;
  for (int c = 0; c < hd; ++c) acc += to_f(op[c]) * to_f(dp[c]);
  const long b = m / T, t = m % T;
  dvec[(b * H + h) * T + t] = acc;
  if (dq_acc)
    for (int c = 0; c < hd; ++c) dq_acc[m * d + h * hd + c] = 0.f;
}

// bf16 version: one warp per token row, 16-byte loads; the lanes holding one
// head's chunks reduce with shuffles.  Also zeroes the dQ accumulator row.
template <int HD>
__global__ void attn_bwd_prep_bf16_kernel(const bf16* o, const bf16* dout,
                                          float* __restrict__ dvec, float* __restrict__ dq_acc, long M, int T,
                                          int H) {
  pdl_start();
  constexpr int CPH = HD / 8;  // 16-byte chunks per head
  const long m = blockIdx.x * (long)(blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const int d = H * HD, nch = d / 8;
  const long b = m / T, t = m % T;
  for (int c0 = 0; c0 < nch; c0 += 32) {
    const int c = c0 + lane;
    float acc = 0.f;
    if (c < nch) {
      uint4 a = *reinterpret_cast<const uint4*>(o + m * d + c * 8);
      uint4 g = *reinterpret_cast<const uint4*>(dout + m * d + c * 8);
      acc = bf16lo(a.x) * bf16lo(g.x) + bf16hi(a.x) * bf16hi(g.x) + bf16lo(a.y) * bf16lo(g.y) +
            bf16hi(a.y) * bf16hi(g.y) + bf16lo(a.z) * bf16lo(g.z) + bf16hi(a.z) * bf16hi(g.z) +
            bf16lo(a.w) * bf16lo(g.w) + bf16hi(a.w) * bf16hi(g.w);
    }
#pragma unroll
    for (int off = 1; off < CPH; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (c < nch && (lane % CPH) == 0) dvec[(b * H + c / CPH) * T + t] = acc;
  }
  float4* z = reinterpret_cast<float4*>(dq_acc + m * d);
  for (int i = lane; i < d / 4; i += 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

template <int HD>
__global__ void __launch_bounds__(128) attn_bwd_kernel(const bf16* qkv,
                                                       const bf16* dout,
                                                       const float* lse,
                                                       const float* dvec,
                                                       bf16* __restrict__ dqkv,
                                                       float* __restrict__ dq_acc, int T, int H,
                                                       float scale, float scale_log2) {
  pdl_start();
  constexpr int BKV = 64, BQ = 64, NC = HD / 8;
  constexpr int TILE = 64 * HD * 2;
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sK = smem_u32(sm);
  const uint32_t sV = sK + TILE;
  const uint32_t sQ = sV + TILE;        // 2 buffers
  const uint32_t sdO = sQ + 2 * TILE;   // 2 buffers
  const uint32_t sDS = sdO + 2 * TILE;  // [64 kv][64 q] bf16, rows of 8 chunks
  float* sL = reinterpret_cast<float*>(sm + 6 * TILE + 64 * 64 * 2);  // [2][64]
  float* sD = sL + 2 * 64;                                              // [2][64]

  const int kvb = blockIdx.x;  // low key blocks have the most query blocks: first
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int d = H * HD;
  const long ld = 3L * d;
  const bf16* Qg = qkv + (long)b * T * ld + h * HD;
  const bf16* Kg = Qg + d;
  const bf16* Vg = Qg + 2 * d;
  const bf16* dOg = dout + (long)b * T * d + h * HD;
  const float* Lg = lse + ((long)b * H + h) * T;
  const float* Dg = dvec + ((long)b * H + h) * T;
  const int kv0 = kvb * BKV;
  const int nq = (T + BQ - 1) / BQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < BKV * NC; i += 128) {
    int r = i / NC, c = i % NC, t = kv0 + r;
    long off = (long)min(t, T - 1) * ld + c * 8;
    int bytes = t < T ? 16 : 0;
    cp_async16(sK + swz<NC>(r, c), Kg + off, bytes);
    cp_async16(sV + swz<NC>(r, c), Vg + off, bytes);
  }
  auto load_q = [&](int qi, int buf) {
    for (int i = threadIdx.x; i < BQ * NC; i += 128) {
      int r = i / NC, c = i % NC, t = qi * BQ + r;
      int bytes = t < T ? 16 : 0;
      int tt = min(t, T - 1);
      cp_async16(sQ + buf * TILE + swz<NC>(r, c), Qg + (long)tt * ld + c * 8, bytes);
      cp_async16(sdO + buf * TILE + swz<NC>(r, c), dOg + (long)tt * d + c * 8, bytes);
    }
    for (int r = threadIdx.x; r < BQ; r += 128) {
      int t = qi * BQ + r;
      sL[buf * 64 + r] = t < T ? Lg[t] * LOG2E_F : INFINITY;
      sD[buf * 64 + r] = t < T ? Dg[t] : 0.f;
    }
  };
  load_q(kvb, 0);
  cp_commit();
  cp_wait<0>();
  __syncthreads();

  uint32_t kfa[HD / 16][4], vfa[HD / 16][4];
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks) {
    ldsm4(kfa[ks], sK + swz<NC>(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)));
    ldsm4(vfa[ks], sV + swz<NC>(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)));
  }
  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  const int kvr_lo = kv0 + warp * 16 + (lane >> 2);

  for (int qi = kvb; qi < nq; ++qi) {
    const int buf = (qi - kvb) & 1;
    if (qi + 1 < nq) load_q(qi + 1, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t qb = sQ + buf * TILE, ob = sdO + buf * TILE;
    const float* Lb = sL + buf * 64;
    const float* Db = sD + buf * 64;
    const int q0 = qi * BQ;

    // S^T = K Q^T (16 keys x 64 queries per warp)
    float st[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) st[n][0] = st[n][1] = st[n][2] = st[n][3] = 0.f;
#pragma unroll
    for (int n2 = 0; n2 < 4; ++n2)
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        uint32_t f[4];
        ldsm4(f, qb + swz<NC>(n2 * 16 + (lane & 7) + ((lane >> 4) << 3), ks * 2 + ((lane >> 3) & 1)));
        mma16816(st[2 * n2], kfa[ks], f[0], f[1]);
        mma16816(st[2 * n2 + 1], kfa[ks], f[2], f[3]);
      }
    // P^T = exp(scale s - lse), zero where query < key or query >= T
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int qc = n * 8 + (lane & 3) * 2 + (e & 1);
        int kr = kvr_lo + (e >> 1) * 8;
        float p = exp2f(st[n][e] * scale_log2 - Lb[qc]);
        if (q0 + qc < kr || q0 + qc >= T || kr >= T) p = 0.f;
        st[n][e] = p;
      }
    // dV += P^T dO
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4] = {pack_bf16x2(st[2 * kk][0], st[2 * kk][1]), pack_bf16x2(st[2 * kk][2], st[2 * kk][3]),
                        pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]),
                        pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3])};
#pragma unroll
      for (int n2 = 0; n2 < HD / 16; ++n2) {
        uint32_t f[4];
        ldsm4t(f, ob + swz<NC>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), n2 * 2 + (lane >> 4)));
        mma16816(dv[2 * n2], pa, f[0], f[1]);
        mma16816(dv[2 * n2 + 1], pa, f[2], f[3]);
      }
    }
    // dP^T = V dO^T
    float dpt[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) dpt[n][0] = dpt[n][1] = dpt[n][2] = dpt[n][3] = 0.f;
#pragma unroll
    for (int n2 = 0; n2 < 4; ++n2)
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        uint32_t f[4];
        ldsm4(f, ob + swz<NC>(n2 * 16 + (lane & 7) + ((lane >> 4) << 3), ks * 2 + ((lane >> 3) & 1)));
        mma16816(dpt[2 * n2], vfa[ks], f[0], f[1]);
        mma16816(dpt[2 * n2 + 1], vfa[ks], f[2], f[3]);
      }
    // dS^T = P^T (dP^T - D)
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int qc = n * 8 + (lane & 3) * 2 + (e & 1);
        st[n][e] = st[n][e] * (dpt[n][e] - Db[qc]);
      }
    // dK += dS^T Q ; and dS^T to shared memory for the dQ product
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4] = {pack_bf16x2(st[2 * kk][0], st[2 * kk][1]), pack_bf16x2(st[2 * kk][2], st[2 * kk][3]),
                        pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]),
                        pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3])};
#pragma unroll
      for (int n2 = 0; n2 < HD / 16; ++n2) {
        uint32_t f[4];
        ldsm4t(f, qb + swz<NC>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), n2 * 2 + (lane >> 4)));
        mma16816(dk[2 * n2], pa, f[0], f[1]);
        mma16816(dk[2 * n2 + 1], pa, f[2], f[3]);
      }
      // rows warp*16 + lane/4 (+8), columns (2kk)*8 + (lane&3)*2 and (2kk+1)*8 + ...
      const int r0 = warp * 16 + (lane >> 2);
      const uint32_t cb = (uint32_t)((lane & 3) * 4);
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(sDS + swz<8>(r0, 2 * kk) + cb), "r"(pa[0]));
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(sDS + swz<8>(r0 + 8, 2 * kk) + cb), "r"(pa[1]));
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(sDS + swz<8>(r0, 2 * kk + 1) + cb), "r"(pa[2]));
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(sDS + swz<8>(r0 + 8, 2 * kk + 1) + cb), "r"(pa[3]));
    }
    __syncthreads();
    // dQ (this warp: queries q0 + warp*16 .. +15) = dS K, reduced into fp32
    float dq[HD / 8][4];
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      ldsm4t(a, sDS + swz<8>(kk * 16 + (lane & 7) + ((lane >> 4) << 3), 2 * warp + ((lane >> 3) & 1)));
#pragma unroll
      for (int n2 = 0; n2 < HD / 16; ++n2) {
        uint32_t f[4];
        ldsm4t(f, sK + swz<NC>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), n2 * 2 + (lane >> 4)));
        mma16816(dq[2 * n2], a, f[0], f[1]);
        mma16816(dq[2 * n2 + 1], a, f[2], f[3]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = q0 + warp * 16 + (lane >> 2) + hh * 8;
      if (t < T) {
        float* dst = dq_acc + ((long)b * T + t) * d + h * HD + (lane & 3) * 2;
#pragma unroll
        for (int n = 0; n < HD / 8; ++n) red_add_v2(dst + n * 8, dq[n][2 * hh] * scale, dq[n][2 * hh + 1] * scale);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int t = kvr_lo + hh * 8;
    if (t < T) {
      bf16* row = dqkv + ((long)b * T + t) * ld + h * HD + (lane & 3) * 2;
#pragma unroll
      for (int n = 0; n < HD / 8; ++n) {
        *reinterpret_cast<uint32_t*>(row + d + n * 8) = pack_bf16x2(dk[n][2 * hh] * scale, dk[n][2 * hh + 1] * scale);
        *reinterpret_cast<uint32_t*>(row + 2 * d + n * 8) = pack_bf16x2(dv[n][2 * hh], dv[n][2 * hh + 1]);
      }
    }
  }
}

// dqkv[m, 0:d] = bf16(sum over key blocks kb <= query block of part[kb][m])
// in key-block order (the deterministic mode of the attention backward)
__global__ void dq_sum_bf16_kernel(const float* part, bf16* __restrict__ dqkv, long M, int T, int d) {
  pdl_start();
  long i = (blockIdx.x * (long)blockDim.x + threadIdx.x) * 4;
  if (i >= M * d) return;
  const long m = i / d;
  const int c = (int)(i % d);
  const int qb = (int)(m % T) / 128;
  float4 acc = *reinterpret_cast<const float4*>(part + i);
  for (int kb = 1; kb <= qb; ++kb) {
    const float4 v = *reinterpret_cast<const float4*>(part + (long)kb * M * d + i);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  *reinterpret_cast<uint2*>(dqkv + m * 3 * d + c) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

// dqkv[:, 0:d] = bf16(dq_acc)
__global__ void dq_to_bf16_kernel(float* __restrict__ dq_acc, bf16* __restrict__ dqkv, long M, int d,
                                  int zero_after) {
  pdl_start();
  long i = (blockIdx.x * (long)blockDim.x + threadIdx.x) * 4;
  if (i >= M * d) return;
  long m = i / d;
  int c = (int)(i % d);
  float4 v = *reinterpret_cast<const float4*>(dq_acc + i);
  uint2 u = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  *reinterpret_cast<uint2*>(dqkv + m * 3 * d + c) = u;
  // the next layer's reduce-adds start from zero
  if (zero_after) *reinterpret_cast<float4*>(dq_acc + i) = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------- fp32 (mode 1) ----

// One CTA of 64 threads per (query t, batch*head).
__global__ void attn_fwd_f32_kernel(const float* qkv, float* __restrict__ o,
                                    float* __restrict__ lse, int T, int H, int hd, float scale) {
  pdl_start();
  extern __shared__ float s[];  // [T] scores, then [64] reduction slots
  float* red = s + T;
  const int t = blockIdx.x, b = blockIdx.y / H, h = blockIdx.y % H;
  const int d = H * hd;
  const long ld = 3L * d;
  const float* q = qkv + ((long)b * T + t) * ld + h * hd;
  const float* kbase = qkv + (long)b * T * ld + d + h * hd;
  const float* vbase = kbase + d;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j <= t; j += blockDim.x) {
    const float* k = kbase + (long)j * ld;
    float acc = 0.f;
    for (int c = 0; c < hd; ++c) acc = fmaf(q[c], k[c], acc);
    acc *= scale;
    s[j] = acc;
    mx = fmaxf(mx, acc);
  }
  red[threadIdx.x] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int i = 1; i < blockDim.x; ++i) m = fmaxf(m, red[i]);
    red[0] = m;
  }
  __syncthreads();
  mx = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j <= t; j += blockDim.x) {
    float p = expf(s[j] - mx);
    s[j] = p;
    sum += p;
  }
  red[threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int i = 0; i < blockDim.x; ++i) a += red[i];
    red[0] = a;
  }
  __syncthreads();
  const float l = red[0];
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j <= t; ++j) acc = fmaf(s[j], vbase[(long)j * ld + c], acc);
    o[((long)b * T + t) * d + h * hd + c] = acc / l;
  }
  if (threadIdx.x == 0) lse[((long)b * H + h) * T + t] = mx + logf(l);
}

// dQ for query t: ds_j = p_j (dO.v_j - D) scale ; dq = sum_j ds_j k_j.
__global__ void attn_bwd_q_f32_kernel(const float* qkv, const float* dout,
                                      const float* lse, const float* dvec,
                                      float* __restrict__ dqkv, int T, int H, int hd, float scale) {
  pdl_start();
  extern __shared__ float s[];
  const int t = blockIdx.x, b = blockIdx.y / H, h = blockIdx.y % H;
  const int d = H * hd;
  const long ld = 3L * d;
  const float* q = qkv + ((long)b * T + t) * ld + h * hd;
  const float* kbase = qkv + (long)b * T * ld + d + h * hd;
  const float* vbase = kbase + d;
  const float* dO = dout + ((long)b * T + t) * d + h * hd;
  const float L = lse[((long)b * H + h) * T + t];
  const float D = dvec[((long)b * H + h) * T + t];
  for (int j = threadIdx.x; j <= t; j += blockDim.x) {
    const float* k = kbase + (long)j * ld;
    const float* v = vbase + (long)j * ld;
    float sc = 0.f, dp = 0.f;
    for (int c = 0; c < hd; ++c) {
      sc = fmaf(q[c], k[c], sc);
      dp = fmaf(dO[c], v[c], dp);
    }
    float p = expf(sc * scale - L);
    s[j] = p * (dp - D) * scale;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j <= t; ++j) acc = fmaf(s[j], kbase[(long)j * ld + c], acc);
    dqkv[((long)b * T + t) * ld + h * hd + c] = acc;
  }
}

// dK, dV for key j: over queries i >= j.
__global__ void attn_bwd_kv_f32_kernel(const float* qkv, const float* dout,
                                       const float* lse, const float* dvec,
                                       float* __restrict__ dqkv, int T, int H, int hd, float scale) {
  pdl_start();
  extern __shared__ float s[];  // p[T], ds[T]
  float* ds = s + T;
  const int j = blockIdx.x, b = blockIdx.y / H, h = blockIdx.y % H;
  const int d = H * hd;
  const long ld = 3L * d;
  const float* qbase = qkv + (long)b * T * ld + h * hd;
  const float* k = qbase + (long)j * ld + d;
  const float* v = k + d;
  const float* dObase = dout + (long)b * T * d + h * hd;
  for (int i = j + threadIdx.x; i < T; i += blockDim.x) {
    const float* q = qbase + (long)i * ld;
    const float* dO = dObase + (long)i * d;
    float sc = 0.f, dp = 0.f;
    for (int c = 0; c < hd; ++c) {
      sc = fmaf(q[c], k[c], sc);
      dp = fmaf(dO[c], v[c], dp);
    }
    float p = expf(sc * scale - lse[((long)b * H + h) * T + i]);
    s[i] = p;
    ds[i] = p * (dp - dvec[((long)b * H + h) * T + i]) * scale;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < hd; c += blockDim.x) {
    float ak = 0.f, av = 0.f;
    for (int i = j; i < T; ++i) {
      ak = fmaf(ds[i], qbase[(long)i * ld + c], ak);
      av = fmaf(s[i], dObase[(long)i * d + c], av);
    }
    float* row = dqkv + ((long)b * T + j) * ld + h * hd + c;
    row[d] = ak;
    row[2 * d] = av;
  }
}

template <int HD>
int launch_fwd(const void* qkv, void* o, float* lse, int B, int T, int H, cudaStream_t st) {
  constexpr int smem = 128 * HD * 2 + 4 * 64 * HD * 2;
  CUDA_TRY(once_per_device((const void*)attn_fwd_kernel<HD>, [](int) {
    return cudaFuncSetAttribute(attn_fwd_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  }));
  dim3 grid((T + 127) / 128, B * H);
  const float scale_log2 = LOG2E_F / sqrtf((float)HD);
  CUDA_TRY(launch_k(attn_fwd_kernel<HD>, grid, 256, smem, st, (const bf16*)qkv, (bf16*)o, lse, T, H, scale_log2));
  LAUNCH_CHECK();
  return GPT2_OK;
}

template <int HD>
int launch_bwd(const void* qkv, const void* dout, const float* lse, const float* dvec, void* dqkv,
               float* dq_acc, int B, int T, int H, cudaStream_t st) {
  constexpr int smem = 6 * 64 * HD * 2 + 64 * 64 * 2 + 4 * 64 * 4;
  CUDA_TRY(once_per_device((const void*)attn_bwd_kernel<HD>, [](int) {
    return cudaFuncSetAttribute(attn_bwd_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  }));
  dim3 grid((T + 63) / 64, B * H);
  const float scale = 1.f / sqrtf((float)HD);
  CUDA_TRY(launch_k(attn_bwd_kernel<HD>, grid, 128, smem, st,
      (const bf16*)qkv, (const bf16*)dout, lse, dvec, (bf16*)dqkv, dq_acc, T, H, scale, scale * LOG2E_F));
  LAUNCH_CHECK();
  return GPT2_OK;
}

}  // namespace

// head_dim 64 runs on the tcgen05 kernels (attention_tc.cu); GPT2_ATTN_FWD=mma
// / GPT2_ATTN_BWD=mma select the warp-level mma.sync kernels instead (a
// diagnostic switch).
static bool env_is_mma(const char* name, int* cache) {
  if (*cache < 0) {
    const char* e = getenv(name);
    *cache = (e && e[0] == 'm') ? 1 : 0;
  }
  return *cache == 1;
}
static bool use_mma_fwd() {
  static int v = -1;
  return env_is_mma("GPT2_ATTN_FWD", &v);
}
static bool use_mma_bwd() {
  static int v = -1;
  return env_is_mma("GPT2_ATTN_BWD", &v);
}

int attn_fwd_bf16(const void* qkv, void* o, float* lse, int B, int T, int H, int hd, cudaStream_t st) {
  if (B <= 0 || T <= 0) return GPT2_OK;
  if (hd == 64 && !use_mma_fwd()) return attn_fwd_tc(qkv, o, lse, B, T, H, st);
  if (hd == 64) return launch_fwd<64>(qkv, o, lse, B, T, H, st);
  if (hd == 16) return launch_fwd<16>(qkv, o, lse, B, T, H, st);
  return GPT2_ERR_UNSUPPORTED_SHAPE;
}

int attn_bwd_bf16(const void* qkv, const void* o, const float* lse, const void* dout, void* dqkv,
                  float* dq_acc, float* dvec, int B, int T, int H, int hd, cudaStream_t st, int dvec_ready,
                  float* dq_part) {
  if (B <= 0 || T <= 0) return GPT2_OK;
  if (hd != 64 && hd != 16) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (dq_part && (hd != 64 || T > 4096)) return GPT2_ERR_UNSUPPORTED_SHAPE;
  const long M = (long)B * T;
  if (!dvec_ready) {
    if (hd == 64)
      CUDA_TRY(launch_k(attn_bwd_prep_bf16_kernel<64>, (unsigned)((M + 7) / 8), 256, 0, st,
          (const bf16*)o, (const bf16*)dout, dvec, dq_acc, M, T, H));
    else
      CUDA_TRY(launch_k(attn_bwd_prep_bf16_kernel<16>, (unsigned)((M + 7) / 8), 256, 0, st,
          (const bf16*)o, (const bf16*)dout, dvec, dq_acc, M, T, H));
    LAUNCH_CHECK();
  }
  int rc = (hd == 64 && (dq_part || !use_mma_bwd()) && T <= 4096)
               ? attn_bwd_tc(qkv, dout, lse, dvec, dqkv, dq_acc, B, T, H, st, dq_part)
               : (hd == 64 ? launch_bwd<64>(qkv, dout, lse, dvec, dqkv, dq_acc, B, T, H, st)
                           : launch_bwd<16>(qkv, dout, lse, dvec, dqkv, dq_acc, B, T, H, st));
  if (rc) return rc;
  const int d = H * hd;
  long n4 = (M * d) / 4;
  if (dq_part) {
    CUDA_TRY(launch_k(dq_sum_bf16_kernel, (unsigned)((n4 + 255) / 256), 256, 0, st, (const float*)dq_part,
                      (bf16*)dqkv, M, T, d));
    LAUNCH_CHECK();
    return GPT2_OK;
  }
  CUDA_TRY(launch_k(dq_to_bf16_kernel, (unsigned)((n4 + 255) / 256), 256, 0, st, dq_acc, (bf16*)dqkv, M, d,
                    dvec_ready));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int attn_fwd_f32(const float* qkv, float* o, float* lse, int B, int T, int H, int hd, cudaStream_t st) {
  if (B <= 0 || T <= 0) return GPT2_OK;
  size_t smem = (size_t)(T + 64) * sizeof(float);
  if (smem > 48 * 1024) return GPT2_ERR_UNSUPPORTED_SHAPE;
  CUDA_TRY(launch_k(attn_fwd_f32_kernel, dim3(T, B * H), 64, smem, st,
      qkv, o, lse, T, H, hd, 1.f / sqrtf((float)hd)));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int attn_bwd_f32(const float* qkv, const float* o, const float* lse, const float* dout, float* dqkv,
                 float* dvec, int B, int T, int H, int hd, cudaStream_t st) {
  if (B <= 0 || T <= 0) return GPT2_OK;
  size_t smem = (size_t)2 * T * sizeof(float);
  if (smem > 48 * 1024) return GPT2_ERR_UNSUPPORTED_SHAPE;
  long rows = (long)B * T * H;
  CUDA_TRY(launch_k(attn_bwd_prep_kernel<float>, (unsigned)((rows + 255) / 256), 256, 0, st,
      o, dout, dvec, nullptr, B, T, H, hd));
  LAUNCH_CHECK();
  const float scale = 1.f / sqrtf((float)hd);
  CUDA_TRY(launch_k(attn_bwd_q_f32_kernel, dim3(T, B * H), 64, (size_t)T * sizeof(float), st,
      qkv, dout, lse, dvec, dqkv, T, H, hd, scale));
  LAUNCH_CHECK();
  CUDA_TRY(launch_k(attn_bwd_kv_f32_kernel, dim3(T, B * H), 64, smem, st,
      qkv, dout, lse, dvec, dqkv, T, H, hd, scale));
  LAUNCH_CHECK();
  return GPT2_OK;
}
