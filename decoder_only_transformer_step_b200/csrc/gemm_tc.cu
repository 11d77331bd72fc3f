// tcgen05 GEMM for sm_100a: the linear layers of the decoder (QKV, attention
// output, MLP fc / proj, tied LM head) and their input- and weight-gradient
// products.  "Pré-treinar um LLM" (compute section) counts each of these as one
// matmul of the forward and two of the same size in the backward; all of them
// are C = A B^T with A and B either K-major or MN-major, which is what this
// kernel takes, so no operand is ever transposed in memory.
//
// Design (persistent over output tiles, one CTA per SM):
//   warp 0      TMA producer: 128B-swizzled tiles of A (128 x 64) and B
//               into a STAGES-deep shared-memory ring (mbarriers).
//   warp 1      allocates TMEM and issues tcgen05.mma (K=16 steps) from one
//               thread; tcgen05.commit frees each ring slot and signals a
//               finished accumulator.
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulator (each warp owns
//               the 32 TMEM lanes = tile rows its warp index allows, and half
//               of the columns), fused bias / residual / GELU / GELU' /
//               fp32-gradient stores.
// The accumulator is double-buffered in TMEM (2 x BN columns), so the
// epilogue of tile i overlaps the main loop of tile i+1.
//
// Two tile shapes: a single CTA computing 128 x BN (BN 128 or 256), and a CTA
// pair (cluster of two SMs) computing 256 x 256 with tcgen05.mma.cta_group::2:
// each CTA loads its 128 rows of A and 128 of the 256 rows of B, so per
// multiply-add each SM moves two thirds of the operand bytes the single-CTA
// 128 x 256 tile needs.  The even CTA issues the MMAs; both run the epilogue
// on their own 128 accumulator rows.  Weight gradients with few output tiles
// are split along K; partial sums go to a workspace and a deterministic
// reduction adds them in split order.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace {

constexpr int BM = 128;
constexpr int BK = 64;               // one 128-byte swizzle row of bf16
constexpr int NUM_EPI_WARPS = 8;  // two per TMEM lane quarter, each owning half the columns
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr uint32_t MN_ATOM_BYTES = 64 * BK * 2;  // one {64 MN x 64 K} TMA box

template <int BN, bool PAIR, bool BIG_EPI>
struct TcCfg {
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;   // output rows per work unit
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;   // rows of B this CTA loads per stage
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  // Per epilogue warp: two 32 x 32 bf16 staging boxes (TMA stores alternate
  // between them) or one 4 KB fp32 box; with BIG_EPI 8 KB, adding a second
  // output's two boxes (GELU) or two boxes for the residual / GELU' operand
  // (TMA loads run one chunk ahead).  The smaller footprint leaves room for
  // a deeper operand ring.
  static constexpr int EPI_WARP_BYTES = BIG_EPI ? 8192 : 4096;
  static constexpr int EPI_BYTES = NUM_EPI_WARPS * EPI_WARP_BYTES;
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

// How the epilogue writes its result.
enum StoreMode : int {
  ST_REG = 0,       // per-thread global stores (general fallback)
  ST_BF16 = 1,      // one bf16 output, TMA store (residual / GELU' operand by TMA load)
  ST_BF16_X2 = 2,   // two bf16 outputs (GELU'(u) and GELU(u)), two TMA stores
  ST_F32 = 3,       // fp32 output, TMA store (beta = 0)
  ST_F32_ADD = 4,   // fp32 output, TMA reduce-add (beta = 1)
  ST_F32_PART = 5,  // fp32 split-K partial [split][M][N], 3-D TMA store
};

struct TcParams {
  int M, N, K;
  int a_mn, b_mn;
  int m_tiles, n_tiles, splits, kb_total;
  int tile_m;  // output rows per work unit (128, or 256 for a CTA pair)
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
// m varies fastest, so consecutive CTAs share the B tile (weights) in L2.
DEVI void decode_unit(const TcParams& p, int u, int& m0, int& nt, int& s, int& kb0, int& kb1) {
  const int mt = u % p.m_tiles;
  const int rest = u / p.m_tiles;
  nt = rest % p.n_tiles;
  s = rest / p.n_tiles;
  m0 = mt * p.tile_m;
  kb0 = (int)((long long)s * p.kb_total / p.splits);
  kb1 = (int)((long long)(s + 1) * p.kb_total / p.splits);
}

enum : int { MODE_PLAIN = 0, MODE_CE = 1 };

// MODE: MODE_PLAIN or MODE_CE (the EPI_CE_FWD epilogue); a separate
// instantiation keeps the cross-entropy state out of the other variants'
// registers.
template <int BN, bool PAIR, bool BIG_EPI, int MODE = MODE_PLAIN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                   const TcParams p) {
  using C = TcCfg<BN, PAIR, BIG_EPI>;
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
  // operand-load barrier of epilogue warp e, buffer b
  auto op_bar = [&](int e, int b) { return bars + 8u * (2 * C::STAGES + 5 + 2 * e + b); };

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
          const uint32_t sa = tiles + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = operand_desc(sa, p.a_mn, k), bd = operand_desc(sb, p.b_mn, k);
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
    // Per 32-column chunk: the residual / GELU' operand box arrives by TMA
    // (issued one chunk ahead), the accumulator comes from TMEM, the result
    // is staged in a 32 x 32 box and written by a TMA store.  Every global
    // access of the epilogue is a TMA box; the threads only touch shared
    // memory and TMEM.
    const int e = warp - 2;
    const int q = warp & 3;              // TMEM lanes [32q, 32q+32) are this warp's
    const int c_begin = (e >> 2) * (BN / 2);
    constexpr int NCH = BN / 64;  // 32-column chunks per warp and tile
    const uint32_t wbox = epi_smem + (uint32_t)e * C::EPI_WARP_BYTES;
    // (the host selects BIG_EPI whenever there is an operand or a second output)
    const bool has_operand =
        BIG_EPI && (p.epi.kind == EPI_BIAS_RESID || p.epi.kind == EPI_DGELU || p.epi.kind == EPI_ROWDOT);
    const bool rowdot = BIG_EPI && p.epi.kind == EPI_ROWDOT;
    int chunk = 0;      // chunks stored by this warp: output box chunk & 1
    int op_issued = 0;  // operand boxes requested: box / barrier k & 1, phase k >> 1
    int op_used = 0;
    // box layout inside the warp's region: bf16 outputs at b * 2048 (and the
    // GELU output at 4096 + b * 2048), operand at 4096 + b * 2048; fp32 at
    // b * 4096 (BIG_EPI) or 0
    auto op_box = [&](int k) { return wbox + 4096u + 2048u * (uint32_t)(k & 1); };
    auto issue_op = [&](int row0_, int col0_) {
      if (lane == 0) {
        const uint32_t bar = op_bar(e, op_issued & 1);
        mbar_arrive_expect_tx(bar, 2048);
        tma_load_2d(op_box(op_issued), &tmC2, bar, col0_, row0_);
      }
      ++op_issued;
    };
    bool ok = true;
    int it = 0;
    constexpr bool ce = MODE == MODE_CE;
    for (int u = unit0; u < units && ok; u += unit_step, ++it) {
      int m0, nt, s, kb0, kb1;
      decode_unit(p, u, m0, nt, s, kb0, kb1);
      const int n0 = nt * BN;
      const int buf = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      const int row0 = m0 + (int)rank * BM + q * 32;
      const int row = row0 + lane;
      // the first chunk's operand does not depend on the accumulator: request
      // it while the MMAs run (every box of the previous tile has been read)
      if (has_operand && p.store != ST_REG && n0 + c_begin < p.N) issue_op(row0, n0 + c_begin);
      if (!mbar_wait_bounded(accf_bar(buf), aph, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // chunks of this warp's columns that lie inside N (warp-uniform)
      const int nch = min(NCH, max(0, (p.N - (n0 + c_begin) + 31) / 32));
      const uint32_t tm_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c_begin);
      // With the small layout TMEM loads run one chunk ahead (chunk ci+1 is
      // requested before chunk ci is processed); the larger epilogues and the
      // cross-entropy epilogue have no registers to spare for that and load
      // each chunk when they reach it.
      constexpr bool PREFETCH = !BIG_EPI && !ce;
      uint32_t r[NCH][32];
      float dsum = 0.f;  // EPI_ROWDOT: this row's sum over the current head's 64 columns
      // EPI_CE_FWD: this row's maximum over the warp's 128 columns (a first
      // pass over TMEM), then exp(acc - max) and its sum in the store pass
      float cmax = -INFINITY, csum = 0.f;
      int ytgt = -1;
      if (ce && nch > 0) {
        // N is a multiple of 128, so a warp's 128 columns are all inside N or
        // all outside: the maximum pass takes two chunks per TMEM wait
        if (row < p.M) ytgt = __ldg(p.epi.ce_tgt + row);
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int ci = 0; ci < NCH; ci += 2) {
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
      if (PREFETCH && nch > 0) tmem_ld_32x32b_x32(tm_row, r[0]);
#pragma unroll
      for (int ci = 0; ci < NCH; ++ci) {
        if (ci >= nch) break;
        const int c = c_begin + 32 * ci;
        const int col0 = n0 + c;
        if (!PREFETCH) tmem_ld_32x32b_x32(tm_row + 32u * (uint32_t)ci, r[ci]);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[ci][j]);
        if (PREFETCH && ci + 1 < NCH && ci + 1 < nch)
          tmem_ld_32x32b_x32(tm_row + 32u * (uint32_t)(ci + 1), r[ci + 1]);
        // (per-element stores are only chosen with the small epilogue layout)
        if (!BIG_EPI && p.store == ST_REG) {
          if (row < p.M) {
            if (col0 + 32 <= p.N) {
              epi_row32_bf16(p.epi, p.partial, s, p.M, p.N, row, col0, v);
            } else {
              // fully unrolled: a runtime-bounded loop would put v in local memory
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < p.N) epi_one<bf16>(p.epi, p.partial, s, p.M, p.N, row, col0 + j, v[j]);
            }
          }
          continue;
        }
        uint4 cur[4];
        if (has_operand) {
          // next chunk's box goes to the other buffer, read one chunk ago
          if (ci + 1 < nch) issue_op(row0, col0 + 32);
          if (!mbar_wait_bounded(op_bar(e, op_used & 1), (uint32_t)(op_used >> 1) & 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          load_bf16_box_row(op_box(op_used), lane, cur);
          ++op_used;
          // these reads precede the TMA load that refills the buffer
          fence_proxy_async_smem();
        }
        epi_apply_row32(p.epi, p.N, col0, v, cur);
        if (ce) {
          constexpr float L2E = 1.4426950408889634f;
          const float cm = cmax * L2E;
          float zv = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            zv = (col0 + j == ytgt) ? v[j] : zv;
            const float ev = ex2_approx(fmaf(v[j], L2E, -cm));
            csum += ev;
            v[j] = ev;
          }
          if (ytgt >= col0 && ytgt < col0 + 32 && row < p.M) p.epi.ce_zt[row] = zv;
        }
        if (rowdot) {
          // the stored (bf16) value times the operand; a head is two chunks
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float t[8];
            unpack8(cur[i], t);
#pragma unroll
            for (int j = 0; j < 8; ++j) dsum = fmaf(__bfloat162float(__float2bfloat16_rn(v[8 * i + j])), t[j], dsum);
          }
          if (ci & 1) {
            if (row < p.M) {
              const int sq = p.epi.seq;
              reinterpret_cast<float*>(p.epi.out2)[((long)(row / sq) * (p.N / 64) + col0 / 64) * sq + row % sq] =
                  dsum;
            }
            dsum = 0.f;
          }
        }
        // the store that last used this chunk's box has read it (two chunks
        // ago; one chunk ago for the single fp32 box of the small layout)
        const bool f32_single = !BIG_EPI && p.store != ST_BF16;
        if (lane == 0) {
          if (f32_single)
            bulk_wait_read<0>();
          else
            bulk_wait_read<1>();
        }
        __syncwarp();
        const uint32_t ob = f32_single ? 0u : (uint32_t)(chunk & 1);
        if (BIG_EPI && p.store == ST_BF16_X2) {
          // v = u: GELU'(u) (saved for the backward) and GELU(u)
          stage_gelu_pair_row(wbox + 2048u * ob, wbox + 4096u + 2048u * ob, lane, v);
        } else if (p.store == ST_BF16 || p.store == ST_BF16_X2) {
          stage_bf16_row(wbox + 2048u * ob, lane, v);
        } else {
          stage_f32_row(wbox + 4096u * ob, lane, v);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          switch (p.store) {
            case ST_BF16:
              tma_store_2d(&tmC, wbox + 2048u * ob, col0, row0);
              break;
            case ST_BF16_X2:
              tma_store_2d(&tmC, wbox + 2048u * ob, col0, row0);
              if (BIG_EPI) tma_store_2d(&tmC2, wbox + 4096u + 2048u * ob, col0, row0);
              break;
            case ST_F32:
              tma_store_2d(&tmC, wbox + 4096u * ob, col0, row0);
              break;
            case ST_F32_ADD:
              tma_reduce_add_2d(&tmC, wbox + 4096u * ob, col0, row0);
              break;
            case ST_F32_PART:
              tma_store_3d(&tmC, wbox + 4096u * ob, col0, row0, s);
              break;
          }
          bulk_commit();
        }
        ++chunk;
      }
      tmem_ld_wait();  // (a no-op unless the loop left early)
      if (!ok) break;
      if (ce && nch > 0 && row < p.M) {
        const long pi = (long)((n0 + c_begin) >> 7) * p.M + row;
        p.epi.ce_max[pi] = cmax;
        p.epi.ce_sum[pi] = csum;
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
      for (int k = op_used; k < op_issued; ++k) mbar_drain_bounded(op_bar(e, k & 1), (uint32_t)(k >> 1) & 1u);
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

// out = beta*out + alpha * sum_s part[s]   (fixed order over s)
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, long mn,
                                     float* __restrict__ out, float alpha, float beta) {
  pdl_start();
  long i = (blockIdx.x * (long)blockDim.x + threadIdx.x) * 4;
  if (i >= mn) return;
  if (i + 4 <= mn) {
    float4 acc = reinterpret_cast<const float4*>(part + i)[0];
    for (int s = 1; s < splits; ++s) {
      float4 t = reinterpret_cast<const float4*>(part + (long)s * mn + i)[0];
      acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
    }
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (beta != 0.f) {
      o = reinterpret_cast<float4*>(out + i)[0];
      o.x *= beta; o.y *= beta; o.z *= beta; o.w *= beta;
    }
    o.x += alpha * acc.x; o.y += alpha * acc.y; o.z += alpha * acc.z; o.w += alpha * acc.w;
    reinterpret_cast<float4*>(out + i)[0] = o;
  } else {
    for (long j = i; j < mn; ++j) {
      float acc = 0.f;
      for (int s = 0; s < splits; ++s) acc += part[(long)s * mn + j];
      out[j] = (beta != 0.f ? beta * out[j] : 0.f) + alpha * acc;
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Tensor map over a row-major tensor: dims[0] is the contiguous (innermost)
// extent in elements, strides are in bytes for dims 1..rank-1.
bool encode_tmap(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t b[3], e[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  CUresult r = enc(tm, dt, rank, const_cast<void*>(base), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 operand [outer, inner] with row pitch `pitch` elements, 128-byte swizzle.
bool make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch,
               uint32_t box_inner, uint32_t box_outer) {
  const uint64_t dims[2] = {inner, outer}, strides[1] = {pitch * 2};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_tmap(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

// [M, N] with pitch ldo in 32 x 32 boxes (epilogue stores and operand loads):
// bf16 with the 64-byte swizzle, fp32 with the 128-byte swizzle (matching
// stage_*_row and load_bf16_box_row).
bool make_out_tmap(CUtensorMap* tm, const void* base, int M, int N, long ldo, bool f32) {
  const uint64_t dims[2] = {(uint64_t)N, (uint64_t)M}, strides[1] = {(uint64_t)ldo * (f32 ? 4 : 2)};
  const uint32_t box[2] = {32, 32};
  return encode_tmap(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2,
                     dims, strides, box, f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int BN, bool PAIR, bool BIG_EPI, int MODE = MODE_PLAIN>
int launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const CUtensorMap& tc2,
              const TcParams& p, int units, cudaStream_t st) {
  using C = TcCfg<BN, PAIR, BIG_EPI>;
  static bool attr_set = false;
  static int max_slots = 0;  // co-resident CTAs (single) or clusters (pairs)
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
  if (!attr_set) {
    CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN, PAIR, BIG_EPI, MODE>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    if (PAIR) {
      cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<BN, PAIR, BIG_EPI, MODE>, &cfg) != cudaSuccess ||
          n <= 0) {
        cudaGetLastError();
        n = num_sms() / 2;
      }
      max_slots = n;
    } else {
      max_slots = num_sms();
    }
    attr_set = true;
  }
  const int slots = units < max_slots ? units : max_slots;
  cfg.gridDim = dim3((PAIR ? 2 : 1) * slots, 1, 1);
  CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, PAIR, BIG_EPI, MODE>, ta, tb, tc, tc2, p));
  LAUNCH_CHECK();
  return GPT2_OK;
}

// Tile choice: bn 0 = automatic (the CTA-pair 256 x 256 tile unless N <= 128),
// 128 / 256 = single-CTA 128 x bn tiles, 512 = the CTA-pair tile.
int resolve_bn(int bn, int N) {
  if (bn == 0) return N <= 128 ? 128 : 512;
  return bn;
}

// Split-K factor for an fp32 (weight-gradient) product with fewer output
// tiles than co-resident CTAs (pairs): the s minimising an estimate of
//   waves(tiles * s) * (k-blocks per unit) * (time of one k-block of a tile)
//   + s * M * N * 8 bytes (partials written and read back) / HBM bandwidth,
// which weighs wave quantisation against the partial-sum traffic.
int auto_splits(int M, int N, int K, int bn) {
  const bool pair = bn == 512;
  const int tile_m = pair ? 2 * BM : BM, tile_n = pair ? 256 : bn;
  const long tiles = (long)((M + tile_m - 1) / tile_m) * ((N + tile_n - 1) / tile_n);
  const int kb = K / BK;
  const int slots = pair ? num_sms() / 2 : num_sms();
  if (tiles >= slots || kb < 8) return 1;
  // one k-block (64 deep) of one tile at ~11 TFLOP/s per SM, in microseconds
  const double kblock_us = 2.0 * 128 * tile_n * BK / 11e6;
  const double bytes_per_us = 6.5e6;  // HBM, bytes per microsecond
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 16 && s <= kb / 4; ++s) {
    const long units = tiles * s;
    const long waves = (units + slots - 1) / slots;
    const double cost = (double)waves * ((double)kb / s) * kblock_us +
                        (s > 1 ? (double)s * M * N * 8.0 / bytes_per_us : 0.0);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

int gemm_tc_set_wait_limit(unsigned long long ns) { return set_unit_wait_limit(ns); }

size_t gemm_tc_split_bytes(int M, int N, int K) {
  int s = auto_splits(M, N, K, resolve_bn(0, N));
  return s > 1 ? (size_t)s * M * N * sizeof(float) : 0;
}

int gemm_tc_bf16(const GemmArgs& g, void* ws, size_t ws_bytes, int bn, int splits, int* err,
                 cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return GPT2_OK;
  if (g.K <= 0 || g.K % BK) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (g.lda % 8 || g.ldb % 8 || g.epi.ldo % 8) return GPT2_ERR_INVALID_ARG;
  if (((uintptr_t)g.A | (uintptr_t)g.B | (uintptr_t)g.epi.out) & 15) return GPT2_ERR_INVALID_ARG;
  bn = resolve_bn(bn, g.N);
  if (bn != 128 && bn != 256 && bn != 512) return GPT2_ERR_INVALID_ARG;
  if (g.epi.kind == EPI_CE_FWD) {
    // 128-column parts: each epilogue warp owns 128 columns of a 256-wide tile
    if (g.N % 128 || !g.epi.ce_max || !g.epi.ce_sum || !g.epi.ce_zt || !g.epi.ce_tgt) return GPT2_ERR_INVALID_ARG;
    if (bn == 128) bn = 256;
  }
  const bool pair = bn == 512;
  const int n_mma = pair ? 256 : bn;  // N of one MMA instruction and of the tile
  const int kb_total = g.K / BK;
  if (splits == 0) splits = g.epi.kind == EPI_F32 ? auto_splits(g.M, g.N, g.K, bn) : 1;
  if (splits > kb_total) splits = kb_total;
  if (splits > 1) {
    if (g.epi.kind != EPI_F32 || g.N % 4 || g.epi.ldo != g.N) return GPT2_ERR_INVALID_ARG;
    size_t need = (size_t)splits * g.M * g.N * sizeof(float);
    if (!ws || ws_bytes < need) splits = 1;
  }

  CUtensorMap ta, tb;
  bool ok_a = g.a_mn ? make_tmap(&ta, g.A, g.M, g.K, g.lda, 64, 64)
                     : make_tmap(&ta, g.A, g.K, g.M, g.lda, 64, BM);
  bool ok_b = g.b_mn ? make_tmap(&tb, g.B, g.N, g.K, g.ldb, 64, 64)
                     : make_tmap(&tb, g.B, g.K, g.N, g.ldb, 64, pair ? n_mma / 2 : n_mma);
  if (!ok_a || !ok_b) return GPT2_ERR_CUDA;

  TcParams p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.a_mn = g.a_mn; p.b_mn = g.b_mn;
  p.tile_m = pair ? 2 * BM : BM;
  p.m_tiles = (g.M + p.tile_m - 1) / p.tile_m;
  p.n_tiles = (g.N + n_mma - 1) / n_mma;
  p.splits = splits;
  p.kb_total = kb_total;
  // instruction descriptor, kind::f16: D fp32 (bit 4), A and B bf16 (bits 7, 10),
  // operand majorness (bits 15, 16), N >> 3 at bit 17, M >> 4 at bit 24 (M = 256
  // for a CTA pair: 128 rows in each CTA).
  p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)g.a_mn << 15) | ((uint32_t)g.b_mn << 16) |
            ((uint32_t)(n_mma >> 3) << 17) | ((uint32_t)(p.tile_m >> 4) << 24);
  p.epi = g.epi;
  p.partial = (float*)ws;
  p.err = err;
  if (splits > 1) p.epi.kind = EPI_F32_PARTIAL;

  // output path: TMA stores of 32 x 32 boxes staged in shared memory
  CUtensorMap tc, tc2;
  memset(&tc, 0, sizeof(tc));
  memset(&tc2, 0, sizeof(tc2));
  bool ok_c = true;
  switch (p.epi.kind) {
    case EPI_STORE:
    case EPI_BIAS:
    case EPI_CE_FWD:
      p.store = ST_BF16;
      ok_c = make_out_tmap(&tc, g.epi.out, g.M, g.N, g.epi.ldo, false);
      break;
    case EPI_ROWDOT:
      if (g.N % 64 || g.epi.seq <= 0 || g.M % g.epi.seq || !g.epi.out2 || ((uintptr_t)g.epi.out2 & 3))
        return GPT2_ERR_INVALID_ARG;
      [[fallthrough]];
    case EPI_BIAS_RESID:
    case EPI_DGELU: {
      // tmC2: the operand read per chunk (same [M, ldo] layout as the output)
      const void* opnd = p.epi.kind == EPI_BIAS_RESID ? g.epi.resid : g.epi.aux;
      if ((uintptr_t)opnd & 15) return GPT2_ERR_INVALID_ARG;
      p.store = ST_BF16;
      ok_c = make_out_tmap(&tc, g.epi.out, g.M, g.N, g.epi.ldo, false) &&
             make_out_tmap(&tc2, opnd, g.M, g.N, g.epi.ldo, false);
      break;
    }
    case EPI_BIAS_GELU:
      if ((uintptr_t)g.epi.out2 & 15) return GPT2_ERR_INVALID_ARG;
      p.store = ST_BF16_X2;
      ok_c = make_out_tmap(&tc, g.epi.out, g.M, g.N, g.epi.ldo, false) &&
             make_out_tmap(&tc2, g.epi.out2, g.M, g.N, g.epi.ldo, false);
      break;
    case EPI_F32:
      if (g.epi.beta == 0.f || g.epi.beta == 1.f) {
        p.store = g.epi.beta == 0.f ? ST_F32 : ST_F32_ADD;
        ok_c = g.epi.ldo % 4 == 0 && make_out_tmap(&tc, g.epi.out, g.M, g.N, g.epi.ldo, true);
      } else {
        p.store = ST_REG;
      }
      break;
    case EPI_F32_PARTIAL: {
      p.store = ST_F32_PART;
      const uint64_t dims[3] = {(uint64_t)g.N, (uint64_t)g.M, (uint64_t)splits};
      const uint64_t strides[2] = {(uint64_t)g.N * 4, (uint64_t)g.M * g.N * 4};
      const uint32_t box[3] = {32, 32, 1};
      ok_c = encode_tmap(&tc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ws, 3, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B);
      break;
    }
    default:
      p.store = ST_REG;
  }
  if (!ok_c) return GPT2_ERR_CUDA;

  const int units = p.m_tiles * p.n_tiles * splits;
  // the second output or the operand boxes need the larger epilogue region
  const bool big = p.store == ST_BF16_X2 || p.epi.kind == EPI_BIAS_RESID || p.epi.kind == EPI_DGELU ||
                   p.epi.kind == EPI_ROWDOT;
  int rc;
  if (p.epi.kind == EPI_CE_FWD) {
    rc = pair ? launch_tc<256, true, false, MODE_CE>(ta, tb, tc, tc2, p, units, st)
              : launch_tc<256, false, false, MODE_CE>(ta, tb, tc, tc2, p, units, st);
  } else if (pair)
    rc = big ? launch_tc<256, true, true>(ta, tb, tc, tc2, p, units, st)
             : launch_tc<256, true, false>(ta, tb, tc, tc2, p, units, st);
  else if (bn == 256)
    rc = big ? launch_tc<256, false, true>(ta, tb, tc, tc2, p, units, st)
             : launch_tc<256, false, false>(ta, tb, tc, tc2, p, units, st);
  else
    rc = big ? launch_tc<128, false, true>(ta, tb, tc, tc2, p, units, st)
             : launch_tc<128, false, false>(ta, tb, tc, tc2, p, units, st);
  if (rc) return rc;
  if (splits > 1) {
    long mn = (long)g.M * g.N;
    long threads = (mn + 3) / 4;
    CUDA_TRY(launch_k(splitk_reduce_kernel, (unsigned)((threads + 255) / 256), 256, 0, st, 
        (const float*)ws, splits, mn, (float*)g.epi.out, g.epi.alpha, g.epi.beta));
    LAUNCH_CHECK();
  }
  return GPT2_OK;
}
