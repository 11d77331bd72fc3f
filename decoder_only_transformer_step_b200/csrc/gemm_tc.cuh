// tcgen05 GEMM kernel for sm_100a: the linear layers of the decoder (QKV,
// attention output, MLP fc / proj, tied LM head) and their input- and
// weight-gradient products.  "Pré-treinar um LLM" (compute section) counts
// each of these as one matmul of the forward and two of the same size in the
// backward; all of them are C = A B^T with A and B either K-major or
// MN-major, which is what this kernel takes, so no operand is ever transposed
// in memory.
//
// Design (persistent over output tiles, one CTA per SM):
//   warp 0      TMA producer: 128B-swizzled tiles of A (128 x 64) and B
//               into a STAGES-deep shared-memory ring (mbarriers).
//   warp 1      allocates TMEM and issues tcgen05.mma (K=16 steps) from one
//               thread; tcgen05.commit frees each ring slot and signals a
//               finished accumulator.
//   warps 2..9  epilogue: each warp owns the 32 TMEM lanes (tile rows) its
//               warp index allows and half of the tile's columns, which it
//               takes 64 at a time ("halves"): one tcgen05.ld wait, the fused
//               arithmetic in packed fp32x2 form, one 32 x 64 box staged in
//               shared memory and written by one TMA store.
// The accumulator is double-buffered in TMEM (2 x BN columns), so the
// epilogue of tile i overlaps the main loop of tile i+1.
//
// The epilogue kind is a template parameter: each instantiation holds only
// its own arithmetic, which keeps the per-tile code short and branch-free.
//
// Two tile shapes: a single CTA computing 128 x BN (BN 128 or 256), and a CTA
// pair (cluster of two SMs) computing 256 x 256 with tcgen05.mma.cta_group::2:
// each CTA loads its 128 rows of A and 128 of the 256 rows of B, so per
// multiply-add each SM moves two thirds of the operand bytes the single-CTA
// 128 x 256 tile needs.  The even CTA issues the MMAs; both run the epilogue
// on their own 128 accumulator rows.  Weight gradients with few output tiles
// are split along K; partial sums go to a workspace and a deterministic
// reduction adds them in split order.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace tcg {

constexpr int BM = 128;
constexpr int BK = 64;            // one 128-byte swizzle row of bf16
constexpr int NUM_EPI_WARPS = 8;  // two per TMEM lane quarter, each owning half the columns
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr uint32_t MN_ATOM_BYTES = 64 * BK * 2;  // one {64 MN x 64 K} TMA box
constexpr uint32_t BOX_BYTES = 4096;             // one 32-row epilogue box: 32 x 64 bf16 or 32 x 32 fp32

// Epilogue staging per warp: the plain bf16 stores (and the cross-entropy
// exponentials) reuse one box per 64-column half; the kinds with an operand
// box (residual, GELU', attention output) or a second output (GELU) and the
// fp32 stores use two.
template <int EK>
struct EpiCfg {
  static constexpr bool ONE_BOX = EK == EPI_STORE || EK == EPI_BIAS || EK == EPI_CE_FWD;
  static constexpr int WARP_BYTES = ONE_BOX ? BOX_BYTES : 2 * BOX_BYTES;
  static constexpr bool OPERAND = EK == EPI_BIAS_RESID || EK == EPI_DGELU || EK == EPI_ROWDOT;
};

template <int BN, bool PAIR, int EK>
struct TcCfg {
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;  // output rows per work unit
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // rows of B this CTA loads per stage
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int NH = BN / 128;  // 64-column halves per warp and tile
  static constexpr int EPI_BYTES = NUM_EPI_WARPS * EpiCfg<EK>::WARP_BYTES;
  // full, empty, acc_full[2], acc_empty[2], drain, operand[8 warps][2]
  static constexpr int NUM_FIXED_BARS = 5 + 2 * NUM_EPI_WARPS;
  static constexpr int STAGES_FIT = (232448 - EPI_BYTES - 1024 - 512) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static constexpr int NUM_BARS = 2 * STAGES + NUM_FIXED_BARS;
  static_assert(NUM_BARS * 8 + 16 <= 512, "barrier region");
  // accumulator-empty arrivals: one per epilogue warp of every CTA of the unit
  static constexpr uint32_t ACCE_COUNT = (PAIR ? 2 : 1) * NUM_EPI_WARPS;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + NUM_BARS * 8 + 16;
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// How the epilogue writes its result (chosen on the host from the kind).
enum StoreMode : int {
  ST_REG = 0,       // fp32 per-thread read-modify-write (beta other than 0 or 1)
  ST_BF16 = 1,      // bf16 32 x 64 boxes, TMA store
  ST_BF16_X2 = 2,   // two bf16 outputs (GELU'(u) and GELU(u)), two TMA stores
  ST_F32 = 3,       // fp32 32 x 32 boxes, TMA store (beta = 0)
  ST_F32_ADD = 4,   // fp32 boxes, TMA reduce-add (beta = 1)
  ST_F32_PART = 5,  // fp32 split-K partial [split][M][N], 3-D TMA store
};

struct TcParams {
  int M, N, K;
  int a_mn, b_mn;
  int m_tiles, n_tiles, splits, kb_total;
  int tile_m;  // output rows per work unit (128, or 256 for a CTA pair)
  int n_fast;  // unit order: n varies fastest (1) or m (0)
  int serial;  // EPI_F32 split along K, reduced in the kernel in split order
  uint32_t idesc;
  int store;
  EpiArgs epi;
  float* partial;
  int* err;
};

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle, sm_100 version 1.
DEVI uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// K-major tile (rows of 64 k = 128 B, 8-row groups 1024 B apart): the k-th
// 16-wide slice starts 32 B further inside the swizzle row.
// MN-major tile ({64 mn x 64 k} boxes 8 KB apart, k rows 128 B apart): the
// k-th 16-row slice starts 2 KB further.
DEVI uint64_t operand_desc(uint32_t tile, int mn_major, int k) {
  return mn_major ? sdesc(tile + k * 2048, MN_ATOM_BYTES, 1024) : sdesc(tile + k * 32, 16, 1024);
}

// Work unit u -> (m tile origin, n tile index, split index, k-block range).
// The units running at one time share the tiles of the larger operand: with
// m fastest, consecutive CTAs load the same B tile and the smaller A is
// re-read from L2; with n fastest the roles swap.  The split index varies
// slowest.
DEVI void decode_unit(const TcParams& p, int u, int& m0, int& nt, int& s, int& kb0, int& kb1) {
  const int tiles = p.m_tiles * p.n_tiles;
  const int t = u % tiles;
  s = u / tiles;
  const int mt = p.n_fast ? t / p.n_tiles : t % p.m_tiles;
  nt = p.n_fast ? t % p.n_tiles : t / p.m_tiles;
  m0 = mt * p.tile_m;
  kb0 = (int)((long long)s * p.kb_total / p.splits);
  kb1 = (int)((long long)(s + 1) * p.kb_total / p.splits);
}

// ---- epilogue pieces: 64 columns of one row, in fp32 pairs ----

DEVI float2 f2(uint32_t lo, uint32_t hi) { return make_float2(__uint_as_float(lo), __uint_as_float(hi)); }
// the two bf16 of a packed word as an fp32 pair (low half first)
DEVI float2 bf2(uint32_t w) { return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); }
DEVI uint32_t pack2(float2 v) { return pack_bf16x2(v.x, v.y); }

// GELU(u) and GELU'(u) of a pair, from one tanh each (tanh form):
//   t = K0 (u + K1 u^3), GELU = u/2 (1 + tanh t),
//   GELU' = 1/2 (1 + tanh t) + u/2 (1 - tanh^2 t) K0 (1 + 3 K1 u^2)
//         = (1/2 + h) + tanh t (1/2 - h tanh t),  h = u/2 K0 (1 + 3 K1 u^2),
// written so that every step is one packed multiply or multiply-add.
DEVI void gelu_pair(float2 u, float2& gelu, float2& grad) {
  const float2 a = __fmul2_rn(u, u);
  const float2 t = __fmul2_rn(u, __ffma2_rn(a, make_float2(GELU_K0 * GELU_K1, GELU_K0 * GELU_K1),
                                            make_float2(GELU_K0, GELU_K0)));
  const float2 th = make_float2(tanh_fast(t.x), tanh_fast(t.y));
  const float2 hu = __fmul2_rn(u, make_float2(0.5f, 0.5f));
  gelu = __ffma2_rn(hu, th, hu);
  // -h, from negated constants
  const float2 hn = __fmul2_rn(hu, __ffma2_rn(a, make_float2(-3.f * GELU_K0 * GELU_K1, -3.f * GELU_K0 * GELU_K1),
                                              make_float2(-GELU_K0, -GELU_K0)));
  const float2 t1 = __ffma2_rn(hn, th, make_float2(0.5f, 0.5f));                      // 1/2 - h tanh t
  const float2 t2 = __ffma2_rn(hn, make_float2(-1.f, -1.f), make_float2(0.5f, 0.5f));  // 1/2 + h
  grad = __ffma2_rn(th, t1, t2);
}

}  // namespace tcg

namespace tcg {

// Bias of columns [c, c + 8) as four fp32 pairs (zero at or past N).  The
// column range is the same for every lane, so the branch is warp-uniform and
// the loads broadcast.
DEVI void bias8(const bf16* bias, int N, int c, float2 (&b)[4]) {
  if (c + 8 <= N) {
    const uint4 u = *reinterpret_cast<const uint4*>(bias + c);
    b[0] = bf2(u.x);
    b[1] = bf2(u.y);
    b[2] = bf2(u.z);
    b[3] = bf2(u.w);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      b[i] = make_float2(c + 2 * i < N ? to_f(bias[c + 2 * i]) : 0.f, c + 2 * i + 1 < N ? to_f(bias[c + 2 * i + 1]) : 0.f);
  }
}

// Shared-memory address of 16-byte slot j of row `lane` in a 128-byte-row box.
DEVI uint32_t box_slot(uint32_t box, int lane, int j) {
  return box + (uint32_t)lane * 128u + 16u * (uint32_t)(j ^ (lane & 7));
}
DEVI uint4 ld_slot(uint32_t addr) {
  uint4 w;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w) : "r"(addr));
  return w;
}

template <int BN, bool PAIR, int EK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                   const TcParams p) {
  using C = TcCfg<BN, PAIR, EK>;
  using E = EpiCfg<EK>;
  static_assert(EK != EPI_CE_FWD || BN == 256, "cross-entropy parts are one warp's 128 columns");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t tiles = (raw + 1023u) & ~1023u;
  uint8_t* tiles_ptr = smem_raw + (tiles - raw);
  const uint32_t epi_smem = tiles + C::STAGES * C::STAGE_BYTES;
  const uint32_t bars = epi_smem + C::EPI_BYTES;
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(tiles_ptr + C::STAGES * C::STAGE_BYTES + C::EPI_BYTES + C::NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (C::STAGES + s); };
  auto accf_bar = [&](int b) { return bars + 8u * (2 * C::STAGES + b); };
  auto acce_bar = [&](int b) { return bars + 8u * (2 * C::STAGES + 2 + b); };
  const uint32_t drain_bar = bars + 8u * (2 * C::STAGES + 4);
  // operand-load barrier of epilogue warp e, half h
  auto op_bar = [&](int e, int h) { return bars + 8u * (2 * C::STAGES + 5 + 2 * e + h); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pairs: consecutive blocks form a cluster; rank 0 issues the MMAs
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int unit_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), C::ACCE_COUNT);
    }
    mbar_init(drain_bar, 1);
    for (int e = 0; e < NUM_EPI_WARPS; ++e) {
      mbar_init(op_bar(e, 0), 1);
      mbar_init(op_bar(e, 1), 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if constexpr (PAIR)
      tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    else
      tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  }
  tc_fence_before();
  __syncthreads();
  // the peer's barriers must be initialised before anything signals them
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // shared memory and TMEM are set up: wait here for the previous kernel
  pdl_start();

  const int units = p.m_tiles * p.n_tiles * p.splits;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer ----
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += unit_step) {
        int m0, nt, s, kb0, kb1;
        decode_unit(p, u, m0, nt, s, kb0, kb1);
        const int ma = m0 + (int)rank * BM;             // this CTA's rows of A
        const int nb = nt * BN + (int)rank * C::B_ROWS;  // this CTA's rows of B
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t sa = tiles + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          if constexpr (PAIR) {
            // both CTAs' bytes are counted on the even CTA's full barrier
            const uint32_t fb = mapa_shared(full_bar(stage), 0);
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
            if (!p.a_mn) {
              tma_load_2d_pair(sa, &tmA, fb, kb * BK, ma);
            } else {
              tma_load_2d_pair(sa, &tmA, fb, ma, kb * BK);
              tma_load_2d_pair(sa + MN_ATOM_BYTES, &tmA, fb, ma + 64, kb * BK);
            }
            if (!p.b_mn) {
              tma_load_2d_pair(sb, &tmB, fb, kb * BK, nb);
            } else {
#pragma unroll
              for (int j = 0; j < C::B_ROWS / 64; ++j)
                tma_load_2d_pair(sb + j * MN_ATOM_BYTES, &tmB, fb, nb + 64 * j, kb * BK);
            }
          } else {
            const uint32_t fb = full_bar(stage);
            mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
            if (!p.a_mn) {
              tma_load_2d(sa, &tmA, fb, kb * BK, ma);
            } else {
              tma_load_2d(sa, &tmA, fb, ma, kb * BK);
              tma_load_2d(sa + MN_ATOM_BYTES, &tmA, fb, ma + 64, kb * BK);
            }
            if (!p.b_mn) {
              tma_load_2d(sb, &tmB, fb, kb * BK, nb);
            } else {
#pragma unroll
              for (int j = 0; j < C::B_ROWS / 64; ++j)
                tma_load_2d(sb + j * MN_ATOM_BYTES, &tmB, fb, nb + 64 * j, kb * BK);
            }
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits (for a
        // pair, the even CTA's full barriers count both CTAs' copies).
        int n = issued < C::STAGES ? issued : C::STAGES;
        for (int i = 1; i <= n; ++i) {
          int s2 = (stage - i + C::STAGES) % C::STAGES;
          uint32_t par = s2 < stage ? phase : (phase ^ 1u);
          if (rank == 0) mbar_drain_bounded(full_bar(s2), par);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------- MMA issuer ----
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued_any = false;
      // Descriptors of stage 0, k-slice 0; the start-address field (bits
      // 0..13, address >> 4) of the others is an add away: every shared-memory
      // address is below 2^18, so the field never carries into the next one.
      const uint64_t a_desc0 = operand_desc(tiles, p.a_mn, 0);
      const uint64_t b_desc0 = operand_desc(tiles + C::A_BYTES, p.b_mn, 0);
      const uint32_t a_kstep = p.a_mn ? 2048u >> 4 : 32u >> 4;
      const uint32_t b_kstep = p.b_mn ? 2048u >> 4 : 32u >> 4;
      for (int u = unit0; u < units && ok; u += unit_step, ++it) {
        int m0, nt, s, kb0, kb1;
        decode_unit(p, u, m0, nt, s, kb0, kb1);
        const int buf = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        const bool acc_free = PAIR ? mbar_wait_bounded_cluster(acce_bar(buf), aph ^ 1u, abort_flag, p.err)
                                   : mbar_wait_bounded(acce_bar(buf), aph ^ 1u, abort_flag, p.err);
        if (!acc_free) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t soff = (uint32_t)stage * (C::STAGE_BYTES >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = a_desc0 + (soff + k * a_kstep), bd = b_desc0 + (soff + k * b_kstep);
            const uint32_t acc = (kb > kb0 || k > 0) ? 1u : 0u;
            if constexpr (PAIR)
              tc_mma_bf16_pair(d_tmem, ad, bd, p.idesc, acc);
            else
              tc_mma_bf16(d_tmem, ad, bd, p.idesc, acc);
          }
          issued_any = true;
          if constexpr (PAIR)
            tc_commit_pair_mask(empty_bar(stage), 3);  // both CTAs' ring slots
          else
            tc_commit(empty_bar(stage));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (PAIR)
          tc_commit_pair_mask(accf_bar(buf), 3);
        else
          tc_commit(accf_bar(buf));
      }
      if (!ok && issued_any) {
        // Wait (bounded) for the MMAs already issued before TMEM is freed.
        if constexpr (PAIR)
          tc_commit_pair(drain_bar);
        else
          tc_commit(drain_bar);
        mbar_drain_bounded(drain_bar, 0);
      }
    }
  } else {
    // ---------------------------------------------------- epilogue ----
    // Per 64-column half: the operand box (residual, GELU' or attention
    // output; requested by TMA before the accumulator wait) or the free
    // staging box, the accumulator from TMEM (two 32-column loads, one wait),
    // the kind's arithmetic on fp32 pairs, the result written into the box
    // and stored by TMA.  Every global access is a TMA box except the bias
    // (a broadcast load) and the row sums of EPI_ROWDOT / EPI_CE_FWD.
    constexpr int NH = C::NH;
    const int e = warp - 2;
    const int q = warp & 3;  // TMEM lanes [32q, 32q+32) are this warp's
    const int c_begin = (e >> 2) * (BN / 2);
    const uint32_t wbox = epi_smem + (uint32_t)e * E::WARP_BYTES;
    const float2 al2 = make_float2(p.epi.alpha, p.epi.alpha);
    int op_issued[2] = {0, 0}, op_used[2] = {0, 0};
    bool ok = true;
    int it = 0;
    for (int u = unit0; u < units && ok; u += unit_step, ++it) {
      int m0, nt, s, kb0, kb1;
      decode_unit(p, u, m0, nt, s, kb0, kb1);
      const int n0 = nt * BN;
      const int buf = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      const int row0 = m0 + (int)rank * BM + q * 32;
      const int row = row0 + lane;
      // halves of this warp's columns that start inside N (warp-uniform)
      const int nh = min(NH, max(0, (p.N - (n0 + c_begin) + 63) / 64));
      if constexpr (E::OPERAND) {
        // the operand boxes do not depend on the accumulator: request them
        // while the MMAs run, once the previous tile's stores have read them
        if (lane == 0) bulk_wait_read<0>();
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < nh) {
            if (lane == 0) {
              const uint32_t bar = op_bar(e, h);
              mbar_arrive_expect_tx(bar, BOX_BYTES);
              tma_load_2d(wbox + BOX_BYTES * h, &tmC2, bar, n0 + c_begin + 64 * h, row0);
            }
            ++op_issued[h];
          }
        }
      }
      if (!mbar_wait_bounded(accf_bar(buf), aph, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tm_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c_begin);

      // Split along K, reduced here in split order: the units of splits
      // 0 .. S-2 store their raw partial tile in their split's slice of the
      // workspace (tmC2) and count it done per (tile, CTA, warp); the unit of
      // the last split, which comes after them in every CTA's unit order,
      // waits for those counts, adds the partials in split order and its own
      // accumulator last, and writes beta * out + alpha * sum through tmC.
      bool serial_done = false;
      if constexpr (EK == EPI_F32) {
        if (p.serial) {
          serial_done = true;
          int* cnt = p.epi.split_cnt + ((u % (p.m_tiles * p.n_tiles)) * (PAIR ? 2 : 1) + (int)rank) * NUM_EPI_WARPS + e;
          const bool last = s + 1 == p.splits;
          if (last) {
            // the earlier splits' partials of this warp's rows and columns
            if (lane == 0) {
              const uint64_t t0 = globaltimer(), lim = g_wait_limit_ns;
              uint32_t spins = 0;
              while (ld_acquire(cnt) < p.splits - 1) {
                if (*abort_flag) {
                  ok = false;
                  break;
                }
                if ((++spins & 63u) == 0 && globaltimer() - t0 > lim) {
                  *abort_flag = 1;
                  if (p.err) atomicOr(p.err, DEV_ERR_TIMEOUT);
                  ok = false;
                  break;
                }
              }
              // the TMA loads below come after that acquire
              fence_proxy_async_global();
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          }
          // 32 columns at a time, alternating between the warp's two boxes
          const int nch = min(2 * NH, max(0, (p.N - (n0 + c_begin) + 31) / 32));
#pragma unroll
          for (int ci = 0; ci < 2 * NH; ++ci) {
            if (!ok || ci >= nch) break;
            const int cc = n0 + c_begin + 32 * ci;
            const uint32_t box = wbox + BOX_BYTES * (uint32_t)(ci & 1);
            // the store that last used this box (two chunks ago) has read it
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            float2 v[16];
            if (last) {
              for (int sp = 0; sp + 1 < p.splits; ++sp) {
                if (lane == 0) {
                  const uint32_t bar = op_bar(e, ci & 1);
                  mbar_arrive_expect_tx(bar, BOX_BYTES);
                  tma_load_3d(box, &tmC2, bar, cc, row0, sp);
                }
                ++op_issued[ci & 1];
                if (!mbar_wait_bounded(op_bar(e, ci & 1), (uint32_t)op_used[ci & 1] & 1u, abort_flag, p.err)) {
                  ok = false;
                  break;
                }
                ++op_used[ci & 1];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const uint4 w4 = ld_slot(box_slot(box, lane, j));
                  const float2 a0 = f2(w4.x, w4.y), a1 = f2(w4.z, w4.w);
                  v[2 * j] = sp == 0 ? a0 : __fadd2_rn(v[2 * j], a0);
                  v[2 * j + 1] = sp == 0 ? a1 : __fadd2_rn(v[2 * j + 1], a1);
                }
                // these reads precede the next TMA write of the box
                fence_proxy_async_smem();
                __syncwarp();
              }
              if (!ok) break;
            }
            uint32_t r[32];
            tmem_ld_32x32b_x32(tm_row + 32u * (uint32_t)ci, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 a = f2(r[2 * i], r[2 * i + 1]);
              v[i] = last ? __fmul2_rn(__fadd2_rn(v[i], a), al2) : a;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(box_slot(box, lane, j), __float_as_uint(v[2 * j].x), __float_as_uint(v[2 * j].y),
                           __float_as_uint(v[2 * j + 1].x), __float_as_uint(v[2 * j + 1].y));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (!last)
                tma_store_3d(&tmC2, box, cc, row0, s);
              else if (p.store == ST_F32)
                tma_store_2d(&tmC, box, cc, row0);
              else
                tma_reduce_add_2d(&tmC, box, cc, row0);
              bulk_commit();
            }
          }
          if (ok && lane == 0) {
            if (!last) {
              // the partial is in memory before it is counted
              bulk_wait_all();
              fence_proxy_async_global();
              red_release_add(cnt, 1);
            } else {
              *cnt = 0;  // ready for the next launch
            }
          }
        }
      }

      // EPI_CE_FWD: this row's maximum over the warp's 128 columns (one
      // cross-entropy part; N is a multiple of 128, so they are all inside N
      // or all outside), then exp(acc - max) and its sum in the store pass
      float cmax = -INFINITY;
      float2 csum2 = make_float2(0.f, 0.f);
      int ytgt = -1;
      if constexpr (EK == EPI_CE_FWD) {
        if (nh > 0) {
          if (row < p.M) ytgt = p.epi.ce_tgt[row];
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int ci = 0; ci < 2 * NH; ci += 2) {
            uint32_t r[2][32];
            tmem_ld_32x32b_x32(tm_row + 32u * (uint32_t)ci, r[0]);
            tmem_ld_32x32b_x32(tm_row + 32u * (uint32_t)(ci + 1), r[1]);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              mx[j & 3] = fmaxf(mx[j & 3], __uint_as_float(r[0][j]));
              mx[j & 3] = fmaxf(mx[j & 3], __uint_as_float(r[1][j]));
            }
          }
          cmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        }
      }
      constexpr float L2E = 1.4426950408889634f;
      const float2 l2e2 = make_float2(L2E, L2E), ncm2 = make_float2(-cmax * L2E, -cmax * L2E);

#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (serial_done || h >= nh) break;
        const int col0 = n0 + c_begin + 64 * h;
        uint32_t r[2][32];
        tmem_ld_32x32b_x32(tm_row + 64u * (uint32_t)h, r[0]);
        tmem_ld_32x32b_x32(tm_row + 64u * (uint32_t)h + 32u, r[1]);
        tmem_ld_wait();
        // the box this half writes: the operand box in place, else the
        // staging box(es), free once the stores that last read them are done
        const uint32_t box = E::OPERAND ? wbox + BOX_BYTES * (uint32_t)h : wbox;
        if constexpr (E::OPERAND) {
          if (!mbar_wait_bounded(op_bar(e, h), (uint32_t)op_used[h] & 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          ++op_used[h];
        } else if (EK != EPI_F32 || p.store != ST_REG) {
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
        }
        if constexpr (EK == EPI_CE_FWD) {
          // the target's logit, if it lies in this half (rare: one lane, one half)
          if (ytgt >= col0 && ytgt < col0 + 64 && row < p.M) {
            float zv = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j) zv = (col0 + j == ytgt) ? __uint_as_float(r[j >> 5][j & 31]) : zv;
            p.epi.ce_zt[row] = zv;
          }
        }
        float2 dacc = make_float2(0.f, 0.f);  // EPI_ROWDOT: this head's row sum, in pairs
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // columns [col0 + 8j, col0 + 8j + 8) as four fp32 pairs
          float2 a[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) a[k] = f2(r[j >> 2][8 * (j & 3) + 2 * k], r[j >> 2][8 * (j & 3) + 2 * k + 1]);
          const int c = col0 + 8 * j;
          const uint32_t sl = box_slot(box, lane, j);
          if constexpr (EK == EPI_STORE) {
#pragma unroll
            for (int k = 0; k < 4; ++k) a[k] = __fmul2_rn(a[k], al2);
            st_shared_v4(sl, pack2(a[0]), pack2(a[1]), pack2(a[2]), pack2(a[3]));
          } else if constexpr (EK == EPI_BIAS) {
            float2 b[4];
            bias8((const bf16*)p.epi.bias, p.N, c, b);
#pragma unroll
            for (int k = 0; k < 4; ++k) a[k] = __fadd2_rn(a[k], b[k]);
            st_shared_v4(sl, pack2(a[0]), pack2(a[1]), pack2(a[2]), pack2(a[3]));
          } else if constexpr (EK == EPI_BIAS_RESID) {
            const uint4 o = ld_slot(sl);
            float2 b[4];
            bias8((const bf16*)p.epi.bias, p.N, c, b);
            a[0] = __fadd2_rn(__fadd2_rn(a[0], b[0]), bf2(o.x));
            a[1] = __fadd2_rn(__fadd2_rn(a[1], b[1]), bf2(o.y));
            a[2] = __fadd2_rn(__fadd2_rn(a[2], b[2]), bf2(o.z));
            a[3] = __fadd2_rn(__fadd2_rn(a[3], b[3]), bf2(o.w));
            st_shared_v4(sl, pack2(a[0]), pack2(a[1]), pack2(a[2]), pack2(a[3]));
          } else if constexpr (EK == EPI_DGELU) {
            const uint4 o = ld_slot(sl);
            a[0] = __fmul2_rn(a[0], bf2(o.x));
            a[1] = __fmul2_rn(a[1], bf2(o.y));
            a[2] = __fmul2_rn(a[2], bf2(o.z));
            a[3] = __fmul2_rn(a[3], bf2(o.w));
            st_shared_v4(sl, pack2(a[0]), pack2(a[1]), pack2(a[2]), pack2(a[3]));
          } else if constexpr (EK == EPI_ROWDOT) {
            // the stored (bf16) value times the operand
            const uint4 o = ld_slot(sl);
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) w[k] = pack2(__fmul2_rn(a[k], al2));
            dacc = __ffma2_rn(bf2(w[0]), bf2(o.x), dacc);
            dacc = __ffma2_rn(bf2(w[1]), bf2(o.y), dacc);
            dacc = __ffma2_rn(bf2(w[2]), bf2(o.z), dacc);
            dacc = __ffma2_rn(bf2(w[3]), bf2(o.w), dacc);
            st_shared_v4(sl, w[0], w[1], w[2], w[3]);
          } else if constexpr (EK == EPI_BIAS_GELU) {
            // u = acc + bias: GELU'(u) into the first box (out), GELU(u) into
            // the second (out2)
            float2 b[4], g[4], d[4];
            bias8((const bf16*)p.epi.bias, p.N, c, b);
#pragma unroll
            for (int k = 0; k < 4; ++k) gelu_pair(__fadd2_rn(a[k], b[k]), g[k], d[k]);
            st_shared_v4(sl, pack2(d[0]), pack2(d[1]), pack2(d[2]), pack2(d[3]));
            st_shared_v4(box_slot(box + BOX_BYTES, lane, j), pack2(g[0]), pack2(g[1]), pack2(g[2]), pack2(g[3]));
          } else if constexpr (EK == EPI_F32) {
#pragma unroll
            for (int k = 0; k < 4; ++k) a[k] = __fmul2_rn(a[k], al2);
            if (p.store == ST_REG) {
              // beta other than 0 or 1: per-element read-modify-write
              if (row < p.M) {
                float* o = (float*)p.epi.out + (long)row * p.epi.ldo;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  if (c + 2 * k < p.N) o[c + 2 * k] = (p.epi.beta != 0.f ? p.epi.beta * o[c + 2 * k] : 0.f) + a[k].x;
                  if (c + 2 * k + 1 < p.N)
                    o[c + 2 * k + 1] = (p.epi.beta != 0.f ? p.epi.beta * o[c + 2 * k + 1] : 0.f) + a[k].y;
                }
              }
            } else {
              // fp32: 32 columns per box, 8 columns = two 16-byte slots
              const uint32_t fb = box + BOX_BYTES * (uint32_t)(j >> 2);
              st_shared_v4(box_slot(fb, lane, 2 * (j & 3)), __float_as_uint(a[0].x), __float_as_uint(a[0].y),
                           __float_as_uint(a[1].x), __float_as_uint(a[1].y));
              st_shared_v4(box_slot(fb, lane, 2 * (j & 3) + 1), __float_as_uint(a[2].x), __float_as_uint(a[2].y),
                           __float_as_uint(a[3].x), __float_as_uint(a[3].y));
            }
          } else if constexpr (EK == EPI_CE_FWD) {
            // exp(acc - max) = 2^(acc log2 e - max log2 e)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 x = __ffma2_rn(a[k], l2e2, ncm2);
              a[k] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              csum2 = __fadd2_rn(csum2, a[k]);
            }
            st_shared_v4(sl, pack2(a[0]), pack2(a[1]), pack2(a[2]), pack2(a[3]));
          }
        }
        if constexpr (EK == EPI_ROWDOT) {
          // one head is one half (N is a multiple of 64)
          if (row < p.M) {
            const int sq = p.epi.seq;
            reinterpret_cast<float*>(p.epi.out2)[((long)(row / sq) * (p.N / 64) + col0 / 64) * sq + row % sq] =
                dacc.x + dacc.y;
          }
        }
        if constexpr (EK == EPI_DGELU) {
          // bias gradient partials: lane l sums columns col0 + 2l, 2l + 1 of
          // the staged (bf16) rows, the values the store writes
          if (p.epi.colsum && row0 < p.M) {
            __syncwarp();
            float2 cs = make_float2(0.f, 0.f);
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) {
              uint32_t wv;
              asm volatile("ld.shared.b32 %0, [%1];"
                           : "=r"(wv)
                           : "r"(box + (uint32_t)rr * 128u + 16u * (uint32_t)((lane >> 2) ^ (rr & 7)) +
                                 4u * (uint32_t)(lane & 3)));
              cs = __fadd2_rn(cs, bf2(wv));
            }
            if (col0 + 2 * lane < p.N)
              *reinterpret_cast<float2*>(p.epi.colsum + (long)(row0 >> 5) * p.N + col0 + 2 * lane) = cs;
          }
        }
        if (EK == EPI_F32 && p.store == ST_REG) continue;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (EK == EPI_BIAS_GELU) {
            tma_store_2d(&tmC, box, col0, row0);
            tma_store_2d(&tmC2, box + BOX_BYTES, col0, row0);
          } else if constexpr (EK == EPI_F32) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              if (col0 + 32 * b >= p.N) break;
              const uint32_t fb = box + BOX_BYTES * (uint32_t)b;
              if (p.store == ST_F32)
                tma_store_2d(&tmC, fb, col0 + 32 * b, row0);
              else if (p.store == ST_F32_ADD)
                tma_reduce_add_2d(&tmC, fb, col0 + 32 * b, row0);
              else
                tma_store_3d(&tmC, fb, col0 + 32 * b, row0, s);
            }
          } else {
            tma_store_2d(&tmC, box, col0, row0);
          }
          bulk_commit();
        }
      }
      tmem_ld_wait();  // (a no-op unless the loop left early)
      if (!ok) break;
      if constexpr (EK == EPI_CE_FWD) {
        if (nh > 0 && row < p.M) {
          const long pi = (long)((n0 + c_begin) >> 7) * p.M + row;
          p.epi.ce_max[pi] = cmax;
          p.epi.ce_sum[pi] = csum2.x + csum2.y;
        }
      }
      // every lane's TMEM loads have completed
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // accumulator-empty barrier of the CTA that issues the MMAs
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(acce_bar(buf), 0));
        else
          mbar_arrive(acce_bar(buf));
      }
    }
    if (lane == 0) {
      bulk_wait_all();
      // operand boxes still in flight (abort path) land before the CTA exits
#pragma unroll
      for (int h = 0; h < 2; ++h)
        for (int k = op_used[h]; k < op_issued[h]; ++k) mbar_drain_bounded(op_bar(e, h), (uint32_t)k & 1u);
    }
    __syncwarp();
  }

  tc_fence_before();
  // After an abort a pair's CTAs cannot observe each other's copies in flight
  // (the odd CTA's loads complete on the even CTA's barriers, which the even
  // CTA drains only for the stages it armed itself): on that error path both
  // wait out a copy's latency many times over before leaving.
  if (PAIR && *abort_flag && (warp == 0 && lane == 0)) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 100000ull) {
    }
  }
  __syncthreads();
  // neither CTA of a pair leaves while the other may still signal its barriers
  if constexpr (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace tcg

namespace tcg {

// Launch one persistent grid (at most one CTA, or CTA pair, per SM).
template <int BN, bool PAIR, int EK>
int launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const CUtensorMap& tc2,
              const TcParams& p, int units, cudaStream_t st) {
  using C = TcCfg<BN, PAIR, EK>;
  static int max_slots_dev[MAX_DEVICES] = {0};  // co-resident CTAs (single) or clusters (pairs)
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (PAIR) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  CUDA_TRY(once_per_device((const void*)gemm_tc_kernel<BN, PAIR, EK>, [&](int dev) -> cudaError_t {
    const cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, PAIR, EK>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int n = num_sms();
    if (PAIR) {
      cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
      if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<BN, PAIR, EK>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms() / 2;
      }
    }
    max_slots_dev[dev < MAX_DEVICES ? dev : 0] = n;
    return cudaSuccess;
  }));
  const int max_slots = max_slots_dev[current_device()];
  const int slots = units < max_slots ? units : max_slots;
  cfg.gridDim = dim3((PAIR ? 2 : 1) * slots, 1, 1);
  CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, PAIR, EK>, ta, tb, tc, tc2, p));
  LAUNCH_CHECK();
  return GPT2_OK;
}

#define TCG_FOR_EACH_KIND(X, BN, PAIR)                                                                   \
  X(BN, PAIR, EPI_STORE) X(BN, PAIR, EPI_BIAS) X(BN, PAIR, EPI_BIAS_RESID) X(BN, PAIR, EPI_BIAS_GELU) \
      X(BN, PAIR, EPI_DGELU) X(BN, PAIR, EPI_F32) X(BN, PAIR, EPI_ROWDOT)

#define TCG_DECLARE(BN, PAIR, EK)                                                                            \
  extern template int launch_tc<BN, PAIR, EK>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, \
                                              const CUtensorMap&, const TcParams&, int, cudaStream_t);
#define TCG_INSTANTIATE(BN, PAIR, EK)                                                                 \
  template int launch_tc<BN, PAIR, EK>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, \
                                       const CUtensorMap&, const TcParams&, int, cudaStream_t);

}  // namespace tcg
