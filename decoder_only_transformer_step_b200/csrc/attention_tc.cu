// Causal self-attention forward on the 5th-generation tensor cores (tcgen05),
// head_dim 64: softmax(q k^T / sqrt(64), keys j <= query i) v per (batch, head).
// The O(T^2) scores of the Kaplan Eq. (2.2) term ("Pré-treinar um LLM") live
// only in tensor memory and registers: per 128-key tile the scores S = Q K^T
// are accumulated in TMEM, one softmax thread per query row turns its row of S
// into probabilities P (bf16, written to shared memory as the next MMA's A
// operand), and O_tile = P V goes back to TMEM; the row's output accumulates in
// registers with the running-max correction (online softmax), and only O and
// the per-row log-sum-exp reach HBM.
//
// One CTA per (batch, head, 128-query block), 320 threads:
//   warp 0      TMA: Q once, K/V tiles into a 2-stage ring (a 3-D tensor map
//               over the packed QKV activation; rows past T read as zeros)
//   warp 1      TMEM allocation; tcgen05.mma S(j) = Q K_j^T (M128 N128 K64) into
//               a double-buffered S, then O_tile(j-1) = P(j-1) V(j-1) (M128 N64
//               K128, V as an MN-major operand) into a double-buffered O_tile
//   warps 2..9  softmax of S(j) (two warps per row group, 64 keys each), P(j)
//               to shared memory, then fold O_tile(j-1) into the registers
// so S(j+1) is computed while the softmax of tile j runs.  Every mbarrier wait
// is bounded; a timeout sets the device status and the CTA drains and exits.
#include <cuda.h>
#include <stdlib.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace {

// 3-D bf16 tensor map, 128-byte swizzle, box {64, 128, 1}.
bool tmap_3d(CUtensorMap* tm, const void* base, const uint64_t* dims, const uint64_t* strides,
             CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint32_t box0 = 64, uint32_t box1 = 128) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]}, s[2] = {strides[0], strides[1]};
  cuuint32_t box[3] = {box0, box1, 1}, e[3] = {1, 1, 1};
  return enc(tm, dt, 3, const_cast<void*>(base), d, s, box, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int HD = 64, BQ = 128, BKV = 128;
constexpr int TILE = 128 * 128;  // one 128-row x 64-col bf16 tile, 128B-swizzled
// forward shared memory: Q (2 buffers: the next work item's Q loads while the
// current one runs; a finished item's O is staged in its Q buffer), a KVS-deep
// K/V ring, P (2 buffers x keys 0-63 | keys 64-127), row max / sum exchange
constexpr int SM_Q = 0;
constexpr int KVS = 3;                    // K/V ring depth: loads run KVS-1 tiles ahead
constexpr int SM_K = SM_Q + 2 * TILE;     // KVS stages
constexpr int SM_V = SM_K + KVS * TILE;   // KVS stages
constexpr int SM_P = SM_V + KVS * TILE;
constexpr int SM_XCHG = SM_P + 4 * TILE;  // [2][2][128] row maxima + [2][128] row sums (floats)
constexpr int SM_TILES = SM_XCHG + 3 * 2 * 128 * 4;
// q_full[2], q_empty[2], kv_full[KVS], kv_empty[KVS], s_full[2], s_free[2], p_full[2], o_full[2], drain,
// xch[4 lane quarters][2] (row-max exchange between the two warps of a quarter),
// row_sync (per-item exchanges of all softmax warps)
constexpr int NUM_BARS = 2 * KVS + 22;
constexpr int SMEM_BYTES = SM_TILES + 1024 + NUM_BARS * 8 + 16;
static_assert(SMEM_BYTES <= 232448, "forward shared memory");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0, O_COL = 256;
constexpr int NUM_THREADS = 320;  // TMA warp, MMA warp, 8 softmax warps

#define LN2_F 0.6931471805599453f
#define LOG2E_F 1.4426950408889634f

DEVI uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16 instruction descriptors: fp32 accumulate, bf16 operands, M = 128.
constexpr uint32_t IDESC_S = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t IDESC_O =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);

DEVI float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Work item of round k for CTA c of G: rounds alternate direction (snake), so
// the long causal items of early rounds and the short ones of late rounds
// even out across CTAs.
DEVI int snake_item(int k, int c, int G) { return k * G + ((k & 1) ? G - 1 - c : c); }

// Persistent: each CTA takes work items (query block, batch, head) in snake
// order over rounds; items are numbered longest causal row first.  Key/value
// blocks are counted globally across a CTA's items (g), so the K/V ring, the
// S / P / O double buffers and their barrier phases run on without a break
// between items.
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmO,
                       float* __restrict__ lse, int T, int H, int n_items, float scale_log2, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + SM_TILES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + SM_TILES + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto q_full = [&](int s) { return bars + 8u * s; };
  auto q_empty = [&](int s) { return bars + 8u * (2 + s); };
  auto kv_full = [&](int s) { return bars + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bars + 8u * (4 + KVS + s); };
  auto s_full = [&](int s) { return bars + 8u * (4 + 2 * KVS + s); };
  auto s_free = [&](int s) { return bars + 8u * (6 + 2 * KVS + s); };
  auto p_full = [&](int s) { return bars + 8u * (8 + 2 * KVS + s); };
  auto o_full = [&](int s) { return bars + 8u * (10 + 2 * KVS + s); };
  const uint32_t drain_bar = bars + 8u * (12 + 2 * KVS);
  auto xch_bar = [&](int q, int s) { return bars + 8u * (13 + 2 * KVS + 2 * q + s); };
  const uint32_t row_sync = bars + 8u * (21 + 2 * KVS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BQ - 1) / BQ;
  const int BH = n_items / nqb;
  const int d = H * HD;
  // work item -> (query block, batch, head); the key blocks are 0..qb
  auto item = [&](int w, int& qb, int& b, int& h) {
    qb = nqb - 1 - w / BH;
    const int bh = w % BH;
    b = bh / H;
    h = bh % H;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(s_free(s), 256);
      mbar_init(p_full(s), 256);
      mbar_init(o_full(s), 1);
    }
    for (int s = 0; s < KVS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(drain_bar, 1);
    for (int qq = 0; qq < 4; ++qq) {
      mbar_init(xch_bar(qq, 0), 64);
      mbar_init(xch_bar(qq, 1), 64);
    }
    mbar_init(row_sync, 256);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmQKV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // shared memory and TMEM are set up: wait here for the previous kernel
  pdl_start();

  if (warp == 0) {
    if (lane == 0) {
      // ----------------------------------------------------------- TMA ----
      bool ok = true;
      int g = 0, it = 0;
      int q_issued = 0, kv_issued = 0;
      for (int k = 0; ok; ++k, ++it) {
        const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
        if (w >= n_items) break;
        int qb, b, h;
        item(w, qb, b, h);
        const int qs = it & 1;
        // the Q buffer was last used by item it-2, whose O store has read it
        if (it >= 2 && !mbar_wait_bounded(q_empty(qs), ((it - 2) >> 1) & 1, abort_flag, err)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full(qs), TILE);
        tma_load_3d(base + SM_Q + qs * TILE, &tmQKV, q_full(qs), h * HD, qb * BQ, b);
        ++q_issued;
        for (int j = 0; j <= qb; ++j, ++g) {
          const int st = g % KVS;
          if (g >= KVS && !mbar_wait_bounded(kv_empty(st), ((g - KVS) / KVS) & 1, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(kv_full(st), 2 * TILE);
          tma_load_3d(base + SM_K + st * TILE, &tmQKV, kv_full(st), d + h * HD, j * BKV, b);
          tma_load_3d(base + SM_V + st * TILE, &tmQKV, kv_full(st), 2 * d + h * HD, j * BKV, b);
          ++kv_issued;
        }
      }
      if (!ok) {
        // let the copies in flight land before the CTA exits
        for (int i = q_issued - 2 < 0 ? 0 : q_issued - 2; i < q_issued; ++i)
          mbar_drain_bounded(q_full(i & 1), (i >> 1) & 1);
        for (int i = kv_issued - KVS < 0 ? 0 : kv_issued - KVS; i < kv_issued; ++i)
          mbar_drain_bounded(kv_full(i % KVS), (i / KVS) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA ----
      bool ok = true;
      bool issued_any = false;
      // O_tile(g) = P(g) V(g) into the O buffer of block g
      auto issue_pv = [&](int gg) -> bool {
        const int pb = gg & 1;
        if (!mbar_wait_bounded(p_full(pb), (gg >> 1) & 1, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t pbase = base + SM_P + pb * 2 * TILE;
        const uint32_t vbase = base + SM_V + (gg % KVS) * TILE;
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          tc_mma_bf16(tmem + O_COL + pb * HD, sdesc(pbase + (k >> 2) * TILE + (k & 3) * 32, 16, 1024),
                      sdesc(vbase + k * 2048, 8192, 1024), IDESC_O, k > 0 ? 1u : 0u);
        tc_commit(o_full(pb));
        tc_commit(kv_empty(gg % KVS));
        return true;
      };
      int g = 0, it = 0;
      for (int k = 0; ok; ++k, ++it) {
        const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
        if (w >= n_items) break;
        int qb, b, h;
        item(w, qb, b, h);
        const int qs = it & 1;
        if (!mbar_wait_bounded(q_full(qs), (it >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qbase = base + SM_Q + qs * TILE;
        for (int j = 0; j <= qb; ++j, ++g) {
          const int st = g % KVS, sb = g & 1;
          if (!mbar_wait_bounded(kv_full(st), (g / KVS) & 1, abort_flag, err)) { ok = false; break; }
          if (g >= 2 && !mbar_wait_bounded(s_free(sb), ((g - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = base + SM_K + st * TILE;
#pragma unroll
          for (int k = 0; k < HD / 16; ++k)
            tc_mma_bf16(tmem + S_COL + sb * BKV, sdesc(qbase + k * 32, 16, 1024), sdesc(kbase + k * 32, 16, 1024),
                        IDESC_S, k > 0 ? 1u : 0u);
          issued_any = true;
          tc_commit(s_full(sb));
          // the previous block's PV (possibly of the previous item) follows
          // this block's S, so softmax of block g overlaps P(g-1) V(g-1)
          if (g >= 1 && !issue_pv(g - 1)) { ok = false; break; }
        }
      }
      if (ok && g >= 1) ok = issue_pv(g - 1);
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_drain_bounded(drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------------------- softmax ----
    // Eight warps: two per TMEM lane quarter, each owning 64 of the 128 key
    // columns of its rows and 32 of the 64 output columns; the two halves of
    // a row exchange partial maxima (per block) and sums (per item) through
    // shared memory.  The per-block maxima are exchanged between the two warps
    // of a lane quarter only (a 64-thread mbarrier per quarter), the per-item
    // steps across all 256 threads; every wait is bounded, so an abort in one
    // warp cannot strand the others.
    const int e = warp - 2;
    const int q = warp & 3;  // TMEM lanes [32q, 32q+32)
    const int half = e >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float* xchg = reinterpret_cast<float*>(base_ptr + SM_XCHG);  // [parity][half][128 rows] maxima
    float* xsum = xchg + 2 * 256;                                 // [half][128 rows] sums
    bool ok = true;
    int g = 0, it = 0;
    for (int k = 0; ok; ++k, ++it) {
      const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
      if (w >= n_items) break;
      int qb, b, h;
      item(w, qb, b, h);
      const int q0 = qb * BQ, grow = q0 + row;
      float m = -INFINITY, l = 0.f, alpha_prev = 1.f;
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      auto fold = [&](int gg, float a) -> bool {
        const int ob = gg & 1;
        if (!mbar_wait_bounded(o_full(ob), (gg >> 1) & 1, abort_flag, err)) return false;
        tc_fence_after();
        uint32_t r0[32];
        tmem_ld_32x32b_x32(tmem + lane_off + O_COL + ob * HD + 32 * half, r0);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = acc[i] * a + __uint_as_float(r0[i]);
        tc_fence_before();
        return true;
      };
      for (int j = 0; j <= qb; ++j, ++g) {
        const int sb = g & 1;
        if (!mbar_wait_bounded(s_full(sb), (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tmem_ld_32x32b_x32(tmem + lane_off + S_COL + sb * BKV + 64 * half + 32 * c, r[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free(sb));
        const bool diag = (j == qb);
        const int kc0 = j * BKV + 64 * half;
        float pmax = m;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float v = __uint_as_float(r[c][i]) * scale_log2;
            if (diag && kc0 + 32 * c + i > grow) v = -INFINITY;
            r[c][i] = __float_as_uint(v);
            pmax = fmaxf(pmax, v);
          }
        float* xp = xchg + sb * 256;
        xp[half * 128 + row] = pmax;
        // only the partner warp (same rows, other 64 keys) is waited for
        mbar_arrive(xch_bar(q, sb));
        if (!mbar_wait_bounded(xch_bar(q, sb), (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
        const float mx = fmaxf(pmax, xp[(1 - half) * 128 + row]);
        const float alpha = ex2(m - mx);
        m = mx;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p = ex2(__uint_as_float(r[c][i]) - m);
            r[c][i] = __float_as_uint(p);
            sum += p;
          }
        l = l * alpha + sum;
        // this half's 64 keys of the P row -> its 128B-swizzled K-major block
        const uint32_t pb = base + SM_P + sb * 2 * TILE + half * TILE + (uint32_t)row * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int gq = c >> 2, o8 = (c & 3) * 8;
          st_shared_v4(pb + 16u * (uint32_t)(c ^ (row & 7)),
                       pack_bf16x2(__uint_as_float(r[gq][o8 + 0]), __uint_as_float(r[gq][o8 + 1])),
                       pack_bf16x2(__uint_as_float(r[gq][o8 + 2]), __uint_as_float(r[gq][o8 + 3])),
                       pack_bf16x2(__uint_as_float(r[gq][o8 + 4]), __uint_as_float(r[gq][o8 + 5])),
                       pack_bf16x2(__uint_as_float(r[gq][o8 + 6]), __uint_as_float(r[gq][o8 + 7])));
        }
        fence_proxy_async_smem();
        mbar_arrive(p_full(sb));
        if (j >= 1 && !fold(g - 1, alpha_prev)) { ok = false; break; }
        alpha_prev = alpha;
      }
      if (ok) ok = fold(g - 1, alpha_prev);
      // row sum = both halves' partial sums (both kept relative to the same m)
      xsum[half * 128 + row] = l;
      mbar_arrive(row_sync);
      if (!mbar_wait_bounded(row_sync, 0, abort_flag, err)) ok = false;
      l += xsum[(1 - half) * 128 + row];
      const int qs = it & 1;
      if (ok) {
        // O / l -> this item's Q buffer (its S MMAs are complete: the last
        // PV, committed after them, has been waited on) -> one TMA store
        const float inv = 1.f / l;
        const uint32_t ob = base + SM_Q + qs * TILE + (uint32_t)row * 128u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(ob + 16u * (uint32_t)((4 * half + c) ^ (row & 7)),
                       pack_bf16x2(acc[8 * c] * inv, acc[8 * c + 1] * inv),
                       pack_bf16x2(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv),
                       pack_bf16x2(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv),
                       pack_bf16x2(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv));
        if (half == 0 && grow < T) lse[((long)b * H + h) * T + grow] = (m + __log2f(l)) * LN2_F;
        fence_proxy_async_smem();
      }
      // all eight softmax warps have staged O (an abort makes every wait
      // return); it also keeps the row-sum exchange of the next item from
      // overwriting a slot before its partner has read it
      mbar_arrive(row_sync);
      if (!mbar_wait_bounded(row_sync, 1, abort_flag, err)) ok = false;
      if (warp == 2 && lane == 0) {
        if (ok && !*abort_flag) {
          tma_store_3d(&tmO, base + SM_Q + qs * TILE, h * HD, q0, b);
          bulk_commit();
          bulk_wait_read<0>();
        }
        mbar_arrive(q_empty(qs));
      }
      __syncwarp();
    }
    if (warp == 2 && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------- forward, two query tiles --
// Persistent; a work item is two consecutive 128-query blocks (2i, 2i+1) of one
// (batch, head), so the K/V tiles are loaded once for both.  Each of the two
// query tiles has its own softmax warpgroup (four warps, one thread per query
// row, so a row's maximum needs no exchange) and its own tensor-memory
// region: S (128 fp32 columns), O (64) and P (64 columns of bf16 pairs).  O is
// accumulated by the tensor cores (P V with P read from tensor memory); a row
// rescales it only when its running maximum grows by more than 2^8, otherwise
// the probabilities are formed against the stale maximum (at most 256, exact
// in the final O / l).  The MMA warp issues S of a tile's next key block right
// after that tile's P V, so one warpgroup's exponentials overlap the other's
// and the tensor-core work of both.
//   warp 0      TMA: both tiles' Q (two item slots), K/V ring
//   warp 1      TMEM allocation, MMA issue
//   warps 4..7  softmax + output of tile 0, warps 8..11 of tile 1
constexpr int F2_KVS = 4;
constexpr int F2_Q = 0;                          // [slot 2][tile 2] Q / O staging
constexpr int F2_K = F2_Q + 4 * TILE;
constexpr int F2_V = F2_K + F2_KVS * TILE;
constexpr int F2_TILES = F2_V + F2_KVS * TILE;
// q_full[2], q_empty[2], kv_full[KVS], kv_empty[KVS], then per tile s_full,
// s_free, p_full, pv_done, o_free, o_staged, and drain
constexpr int F2_NUM_BARS = 4 + 2 * F2_KVS + 12 + 1;
constexpr int F2_SMEM = F2_TILES + 1024 + F2_NUM_BARS * 8 + 16;
static_assert(F2_SMEM <= 232448, "forward shared memory");
constexpr float F2_RESCALE = 8.f;  // log2 of the largest un-rescaled probability
// Twelve warps in three warpgroups: WG0 = TMA (warp 0), MMA (warp 1), two idle
// warps; WG1 / WG2 = the softmax of query tile 0 / 1.  Register budgets after
// setmaxnreg: with 168 per thread at launch the block owns 384 x 168 = 64512,
// split as 128 x 80 + 256 x 208 = 63488.
constexpr int F2_THREADS = 384;
constexpr int F2_LAUNCH_REGS = 168, F2_REGS_CTRL = 80, F2_REGS_SOFT = 208;
static_assert(128 * F2_REGS_CTRL + 256 * F2_REGS_SOFT <= F2_THREADS * F2_LAUNCH_REGS, "register split");

template <int N> DEVI void reg_dealloc() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N> DEVI void reg_alloc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// max(a, b, c): the three-operand form of max.f32 (NaN operands are
// ignored as by fmaxf), half the instructions of a pairwise row maximum.
DEVI float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__global__ void __launch_bounds__(F2_THREADS, 1)
    attn_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmO,
                        float* __restrict__ lse, int T, int H, int n_items, float scale_log2, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + F2_TILES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + F2_TILES + F2_NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto q_full = [&](int s) { return bars + 8u * s; };
  auto q_empty = [&](int s) { return bars + 8u * (2 + s); };
  auto kv_full = [&](int s) { return bars + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bars + 8u * (4 + F2_KVS + s); };
  // per-tile barriers: k = 0 s_full, 1 s_free, 2 p_full, 3 pv_done, 4 o_free, 5 o_staged
  auto tbar = [&](int t, int k) { return bars + 8u * (4 + 2 * F2_KVS + 6 * t + k); };
  const uint32_t drain_bar = bars + 8u * (4 + 2 * F2_KVS + 12);
  auto qbuf = [&](int slot, int t) { return base + F2_Q + (uint32_t)(2 * slot + t) * TILE; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BQ - 1) / BQ;
  const int npairs = (nqb + 1) / 2;
  const int BH = n_items / npairs;
  const int d = H * HD;
  // work item -> (first query block, batch, head); longest items first
  auto item = [&](int w, int& qa, int& b, int& h) {
    qa = 2 * (npairs - 1 - w / BH);
    const int bh = w % BH;
    b = bh / H;
    h = bh % H;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 2);  // one arrival per softmax warpgroup
    }
    for (int s = 0; s < F2_KVS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(tbar(t, 0), 1);
      mbar_init(tbar(t, 1), 4);
      mbar_init(tbar(t, 2), 4);
      mbar_init(tbar(t, 3), 1);
      mbar_init(tbar(t, 4), 4);
      mbar_init(tbar(t, 5), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmQKV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_start();

  if (warp < 4) {
   reg_dealloc<F2_REGS_CTRL>();
   if (warp == 0) {
    if (lane == 0) {
      // ----------------------------------------------------------- TMA ----
      bool ok = true;
      int g = 0, it = 0, q_issued = 0, kv_issued = 0;
      for (int k = 0; ok; ++k, ++it) {
        const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
        if (w >= n_items) break;
        int qa, b, h;
        item(w, qa, b, h);
        const bool hasb = qa + 1 < nqb;
        const int nkb = hasb ? qa + 2 : qa + 1;
        const int slot = it & 1;
        // both Q buffers of the slot were last used by item it-2, whose O
        // stores have read them
        if (it >= 2 && !mbar_wait_bounded(q_empty(slot), ((it - 2) >> 1) & 1, abort_flag, err)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full(slot), (hasb ? 2 : 1) * TILE);
        tma_load_3d(qbuf(slot, 0), &tmQKV, q_full(slot), h * HD, qa * BQ, b);
        if (hasb) tma_load_3d(qbuf(slot, 1), &tmQKV, q_full(slot), h * HD, (qa + 1) * BQ, b);
        ++q_issued;
        for (int j = 0; j < nkb; ++j, ++g) {
          const int st = g % F2_KVS;
          if (g >= F2_KVS && !mbar_wait_bounded(kv_empty(st), ((g - F2_KVS) / F2_KVS) & 1, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(kv_full(st), 2 * TILE);
          tma_load_3d(base + F2_K + st * TILE, &tmQKV, kv_full(st), d + h * HD, j * BKV, b);
          tma_load_3d(base + F2_V + st * TILE, &tmQKV, kv_full(st), 2 * d + h * HD, j * BKV, b);
          ++kv_issued;
        }
      }
      if (!ok) {
        for (int i = q_issued - 2 < 0 ? 0 : q_issued - 2; i < q_issued; ++i)
          mbar_drain_bounded(q_full(i & 1), (i >> 1) & 1);
        for (int i = kv_issued - F2_KVS < 0 ? 0 : kv_issued - F2_KVS; i < kv_issued; ++i)
          mbar_drain_bounded(kv_full(i % F2_KVS), (i / F2_KVS) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA ----
      bool ok = true, issued_any = false;
      int nS[2] = {0, 0}, nP[2] = {0, 0}, nI[2] = {0, 0};
      int g0 = 0, it = 0, kv_ready = 0;  // K/V blocks (counted over items) known to have landed
      for (int k = 0; ok; ++k, ++it) {
        const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
        if (w >= n_items) break;
        int qa, b, h;
        item(w, qa, b, h);
        const bool hasb = qa + 1 < nqb;
        const int nkb = hasb ? qa + 2 : qa + 1;
        const int slot = it & 1;
        if (!mbar_wait_bounded(q_full(slot), (it >> 1) & 1, abort_flag, err)) { ok = false; break; }
        auto issue_s = [&](int t, int j) -> bool {
          const int gg = g0 + j;
          while (kv_ready <= gg) {
            if (!mbar_wait_bounded(kv_full(kv_ready % F2_KVS), (kv_ready / F2_KVS) & 1, abort_flag, err))
              return false;
            ++kv_ready;
          }
          // the softmax has loaded this tile's previous S
          if (nS[t] >= 1 && !mbar_wait_bounded(tbar(t, 1), (nS[t] - 1) & 1, abort_flag, err)) return false;
          tc_fence_after();
          const uint32_t qb = qbuf(slot, t), kb = base + F2_K + (gg % F2_KVS) * TILE;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc_mma_bf16(tmem + 256u * t, sdesc(qb + kk * 32, 16, 1024), sdesc(kb + kk * 32, 16, 1024), IDESC_S,
                        kk > 0 ? 1u : 0u);
          tc_commit(tbar(t, 0));
          ++nS[t];
          issued_any = true;
          return true;
        };
        auto issue_pv = [&](int t, int j) -> bool {
          if (!mbar_wait_bounded(tbar(t, 2), nP[t] & 1, abort_flag, err)) return false;
          // the first block of an item overwrites O: the previous item's
          // output must have been read out of tensor memory
          if (j == 0 && nI[t] >= 1 && !mbar_wait_bounded(tbar(t, 4), (nI[t] - 1) & 1, abort_flag, err))
            return false;
          tc_fence_after();
          const uint32_t vb = base + F2_V + ((g0 + j) % F2_KVS) * TILE;
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            tc_mma_bf16_ts(tmem + 256u * t + 128u, tmem + 256u * t + 192u + 8u * kk, sdesc(vb + kk * 2048, 8192, 1024),
                           IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(tbar(t, 3));
          ++nP[t];
          return true;
        };
        // S of a tile's next key block needs only that the softmax has
        // loaded the current S (P lives in other columns), so it is issued
        // ahead of the current block's P V: the softmax finds the next S
        // ready as soon as it has released the current P
        ok = issue_s(0, 0) && (!hasb || issue_s(1, 0));
        for (int j = 0; j < nkb && ok; ++j) {
          if (j + 1 <= qa && !issue_s(0, j + 1)) { ok = false; break; }
          if (hasb && j + 1 < nkb && !issue_s(1, j + 1)) { ok = false; break; }
          if (j <= qa && !issue_pv(0, j)) { ok = false; break; }
          if (hasb && !issue_pv(1, j)) { ok = false; break; }
          // every MMA reading this K/V slot has been issued
          tc_commit(kv_empty((g0 + j) % F2_KVS));
        }
        ++nI[0];
        if (hasb) ++nI[1];
        g0 += nkb;
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_drain_bounded(drain_bar, 0);
      }
    }
   }
  } else {
    reg_alloc<F2_REGS_SOFT>();
    // ------------------------------------------------- softmax, output ----
    const int t = (warp - 4) >> 2;  // query tile of this warpgroup
    const int q = warp & 3;         // TMEM lanes [32q, 32q+32)
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tS = tmem + lane_off + 256u * t, tO = tS + 128u, tP = tS + 192u;
    const bool leader = (warp & 3) == 0 && lane == 0;  // first warp of the warpgroup
    bool ok = true;
    int ns = 0, np = 0, nit = 0;
    for (int k = 0; ok; ++k) {
      const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
      if (w >= n_items) break;
      int qa, b, h;
      item(w, qa, b, h);
      const int slot = k & 1;
      const int qt = qa + t;  // this tile's query block
      if (qt >= nqb) {
        // tile 1 absent (an odd number of query blocks): nothing to compute.
        // Its release of the Q slot must not run ahead into a later phase of
        // the slot's barrier, so it waits until this item's Q has landed
        // (which the producer issues only after the slot's previous phase).
        if (leader) {
          if (!mbar_wait_bounded(q_full(slot), (k >> 1) & 1, abort_flag, err)) ok = false;
          mbar_arrive(q_empty(slot));
        }
        __syncwarp();
        continue;
      }
      const int grow = qt * BQ + row;
      float m_use = -INFINITY, l = 0.f;
      for (int j = 0; j <= qt; ++j) {
        if (!mbar_wait_bounded(tbar(t, 0), ns & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + 32u * c, v[c]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tbar(t, 1));
        ++ns;
        // raw scores; keys past the query masked on the diagonal block.  The
        // row maximum runs as eight independent chains (one dependent chain
        // of 128 would cost its latency 128 times).
        float mxs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mxs[i] = -INFINITY;
        if (j == qt) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float x = (32 * c + i > row) ? -INFINITY : __uint_as_float(v[c][i]);
              v[c][i] = __float_as_uint(x);
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mxs[(i >> 1) & 7] = fmax3(mxs[(i >> 1) & 7], __uint_as_float(v[c][i]), __uint_as_float(v[c][i + 1]));
        const float mx = fmaxf(fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3])),
                               fmaxf(fmaxf(mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7])));
        const float m_new = fmaxf(m_use, mx * scale_log2);
        float alpha = 1.f;
        bool resc = false;
        if (j == 0) {
          m_use = m_new;
        } else if (m_new > m_use + F2_RESCALE) {
          alpha = ex2(m_use - m_new);
          m_use = m_new;
          resc = true;
        }
        // probabilities (bf16 pairs) in registers first; the previous P V
        // is waited for only before they are stored over its P
        // two columns per packed fp32x2 multiply-add and add
        float2 sums[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_use, -m_use);
        uint32_t pk[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[c][2 * i]), __uint_as_float(v[c][2 * i + 1])),
                                        sc2, nm2);
            const float2 pr = make_float2(ex2(x.x), ex2(x.y));
            sums[i & 1] = __fadd2_rn(sums[i & 1], pr);
            pk[c][i] = pack_bf16x2(pr.x, pr.y);
          }
        l = l * alpha + ((sums[0].x + sums[0].y) + (sums[1].x + sums[1].y));
        // P V of the previous block has finished reading P and writing O
        if (np >= 1 && !mbar_wait_bounded(tbar(t, 3), (np - 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st_32x32b_x16(tP + 16u * c, pk[c]);
        if (__any_sync(0xffffffffu, resc)) {
          // rare: this warp's rows whose maximum grew rescale their O
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tO + 32u * hh, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_32x32b_x32(tO + 32u * hh, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tbar(t, 2));
        ++np;
      }
      if (!ok) break;
      // ---- output: O / l in bf16 through this tile's Q buffer, one TMA store
      if (!mbar_wait_bounded(tbar(t, 3), (np - 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      uint32_t o[2][32];
      tmem_ld_32x32b_x32(tO, o[0]);
      tmem_ld_32x32b_x32(tO + 32u, o[1]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tbar(t, 4));
      const float inv = 1.f / l;
      const uint32_t ob = qbuf(slot, t) + (uint32_t)row * 128u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t* oc = &o[c >> 2][(c & 3) * 8];
        st_shared_v4(ob + 16u * (uint32_t)(c ^ (row & 7)),
                     pack_bf16x2(__uint_as_float(oc[0]) * inv, __uint_as_float(oc[1]) * inv),
                     pack_bf16x2(__uint_as_float(oc[2]) * inv, __uint_as_float(oc[3]) * inv),
                     pack_bf16x2(__uint_as_float(oc[4]) * inv, __uint_as_float(oc[5]) * inv),
                     pack_bf16x2(__uint_as_float(oc[6]) * inv, __uint_as_float(oc[7]) * inv));
      }
      if (grow < T) lse[((long)b * H + h) * T + grow] = (m_use + __log2f(l)) * LN2_F;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(tbar(t, 5));
      if (!mbar_wait_bounded(tbar(t, 5), nit & 1, abort_flag, err)) { ok = false; break; }
      ++nit;
      if (leader) {
        tma_store_3d(&tmO, qbuf(slot, t), h * HD, qt * BQ, b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(q_empty(slot));
      }
      __syncwarp();
    }
    if (leader) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ----------------------------------------------------------------- backward --
// One CTA per (batch, head, 128-key block), looping over the query blocks at or
// below the diagonal.  Per query block t:
//   S^T = K Q^T and dP^T = V dO^T          (M128 N128 K64, into TMEM)
//   P^T = exp(scale S^T - LSE), dS^T = P^T (dP^T - D)   (elementwise warps)
//   dV += P^T dO, dK += dS^T Q              (M128 N64 K128, TMEM accumulators)
//   dQ  = dS K                              (A = the dS^T buffer read MN-major)
// and dQ is added into an fp32 buffer by TMA reductions (staged through the
// block's spent Q/dO ring slot).  Eight elementwise warps (two per TMEM
// lane quarter, 64 of the 128 query columns each) need no row reductions here,
// so they split the columns with no communication; the next block's S^T/dP^T
// MMAs run while they work.
constexpr int QS = 3;  // Q/dO ring depth: loads run QS-1 query blocks ahead
constexpr int BS_K = 0, BS_V = TILE, BS_Q = 2 * TILE, BS_DO = BS_Q + QS * TILE, BS_P = BS_DO + QS * TILE;
constexpr int BS_DS = BS_P + 2 * TILE;
constexpr int BS_MAX_QBLOCKS = 32;  // T <= 4096
constexpr int BS_LD = BS_DS + 2 * TILE;  // [query block][LSE x128 | D x128] floats
constexpr int BS_TILES = BS_LD + BS_MAX_QBLOCKS * 256 * 4;
// kv_full, qdo_full[QS], qdo_empty[QS], st_full, st_free, ps_full, mma2_done, drain, tail
constexpr int B_NUM_BARS = 2 * QS + 7;
constexpr int B_SMEM_BYTES = BS_TILES + 1024 + B_NUM_BARS * 8 + 16;
constexpr int B_NUM_THREADS = 320;
// dQ is double-buffered (C_DQ + 64 * (t & 1)) so block t's MMAs never wait for
// block t-1's dQ to be drained.
constexpr uint32_t C_ST = 0, C_DPT = 128, C_DV = 256, C_DK = 320, C_DQ = 384;
// dQ = dS K: both operands read MN-major
constexpr uint32_t IDESC_DQ =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);

__global__ void __launch_bounds__(B_NUM_THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDQKV,
                       const float* lse, const float* dvec, int T, int H, float scale,
                       float scale_log2, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  float* sLD = reinterpret_cast<float*>(base_ptr + BS_LD);
  const uint32_t bars = base + BS_TILES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + BS_TILES + B_NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t kv_full = bars;
  auto qdo_full = [&](int s) { return bars + 8u * (1 + s); };
  auto qdo_empty = [&](int s) { return bars + 8u * (1 + QS + s); };
  const uint32_t st_full = bars + 8u * (1 + 2 * QS), st_free = bars + 8u * (2 + 2 * QS);
  const uint32_t ps_full = bars + 8u * (3 + 2 * QS);
  const uint32_t mma2_done = bars + 8u * (4 + 2 * QS), drain_bar = bars + 8u * (5 + 2 * QS);
  const uint32_t tail_bar = bars + 8u * (6 + 2 * QS);  // dK/dV staged by all eight elementwise warps

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = (T + BQ - 1) / BQ;
  const int kvb = blockIdx.x;  // low key blocks have the most query blocks: first
  const int b = blockIdx.y / H, h = blockIdx.y % H;
  const int d = H * HD;
  const int kv0 = kvb * BKV;
  const int nblk = nq - kvb;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(qdo_full(s), 1);
      // released by the MMAs of the block and by the eight elementwise warps
      // once their dQ reduction has read the slot
      mbar_init(qdo_empty(s), 1 + 8);
    }
    mbar_init(st_full, 1);
    mbar_init(st_free, 256);
    mbar_init(ps_full, 256);
    mbar_init(mma2_done, 1);
    mbar_init(drain_bar, 1);
    mbar_init(tail_bar, 256);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmQKV);
    tma_prefetch_desc(&tmDO);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // shared memory and TMEM are set up: wait here for the previous kernel
  pdl_start();

  if (warp == 0) {
    if (lane == 0) {
      // ----------------------------------------------------------- TMA ----
      int issued = 0;
      bool ok = true;
      mbar_arrive_expect_tx(kv_full, 2 * TILE);
      tma_load_3d(base + BS_K, &tmQKV, kv_full, d + h * HD, kv0, b);
      tma_load_3d(base + BS_V, &tmQKV, kv_full, 2 * d + h * HD, kv0, b);
      for (int t = 0; t < nblk; ++t) {
        const int buf = t % QS;
        if (t >= QS && !mbar_wait_bounded(qdo_empty(buf), ((t - QS) / QS) & 1, abort_flag, err)) {
          ok = false;
          break;
        }
        const int q0 = (kvb + t) * BQ;
        mbar_arrive_expect_tx(qdo_full(buf), 2 * TILE);
        tma_load_3d(base + BS_Q + buf * TILE, &tmQKV, qdo_full(buf), h * HD, q0, b);
        tma_load_3d(base + BS_DO + buf * TILE, &tmDO, qdo_full(buf), h * HD, q0, b);
        ++issued;
      }
      if (!ok) {
        mbar_drain_bounded(kv_full, 0);
        for (int t = issued - QS < 0 ? 0 : issued - QS; t < issued; ++t)
          mbar_drain_bounded(qdo_full(t % QS), (t / QS) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA ----
      bool ok = mbar_wait_bounded(kv_full, 0, abort_flag, err);
      bool issued_any = false;
      auto issue_s = [&](int t) -> bool {
        const int buf = t % QS;
        if (!mbar_wait_bounded(qdo_full(buf), (t / QS) & 1, abort_flag, err)) return false;
        if (t >= 1 && !mbar_wait_bounded(st_free, (t - 1) & 1, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t qb = base + BS_Q + buf * TILE, ob = base + BS_DO + buf * TILE;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k)
          tc_mma_bf16(tmem + C_ST, sdesc(base + BS_K + k * 32, 16, 1024), sdesc(qb + k * 32, 16, 1024), IDESC_S,
                      k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k)
          tc_mma_bf16(tmem + C_DPT, sdesc(base + BS_V + k * 32, 16, 1024), sdesc(ob + k * 32, 16, 1024), IDESC_S,
                      k > 0 ? 1u : 0u);
        issued_any = true;
        tc_commit(st_full);
        return true;
      };
      auto issue_mma2 = [&](int t) -> bool {
        const int buf = t % QS;
        if (!mbar_wait_bounded(ps_full, t & 1, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t qb = base + BS_Q + buf * TILE, ob = base + BS_DO + buf * TILE;
#pragma unroll
        for (int k = 0; k < BQ / 16; ++k)
          tc_mma_bf16(tmem + C_DV, sdesc(base + BS_P + (k >> 2) * TILE + (k & 3) * 32, 16, 1024),
                      sdesc(ob + k * 2048, 8192, 1024), IDESC_O, (t > 0 || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < BQ / 16; ++k)
          tc_mma_bf16(tmem + C_DK, sdesc(base + BS_DS + (k >> 2) * TILE + (k & 3) * 32, 16, 1024),
                      sdesc(qb + k * 2048, 8192, 1024), IDESC_O, (t > 0 || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          tc_mma_bf16(tmem + C_DQ + 64 * (t & 1), sdesc(base + BS_DS + k * 2048, TILE, 1024),
                      sdesc(base + BS_K + k * 2048, 8192, 1024), IDESC_DQ, k > 0 ? 1u : 0u);
        tc_commit(mma2_done);
        tc_commit(qdo_empty(buf));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int t = 0; t < nblk && ok; ++t) {
        if (t + 1 < nblk && !issue_s(t + 1)) { ok = false; break; }
        if (!issue_mma2(t)) { ok = false; break; }
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_drain_bounded(drain_bar, 0);
      }
    }
  } else {
    // -------------------------------------------- elementwise + dQ drain ----
    const int e = warp - 2;
    const int q = warp & 3;    // TMEM lanes [32q, 32q+32)
    const int half = e >> 2;   // query columns [64*half, 64*half+64)
    const int row = q * 32 + lane;
    const int kv = kv0 + row;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int tid = threadIdx.x - 64;
    bool ok = true;
    auto drain_dq = [&](int t) {
      // dQ rows are queries of block t; this warp takes 32 of the 64 columns.
      // Block t's Q/dO ring slot (its MMAs are complete) holds the fp32 dQ
      // tile as two 128-row x 32-column boxes in the 128-byte swizzle; each
      // warp stages its 32 x 32 part and adds it to dq_acc with one TMA
      // reduce, then releases the slot to the loads.
      const int sl = t % QS;
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem + lane_off + C_DQ + 64 * (t & 1) + 32 * half, r);
      tmem_ld_wait();
      const uint32_t box = base + (half ? BS_DO : BS_Q) + sl * TILE + (uint32_t)(q * 32) * 128u;
      const uint32_t rb = box + (uint32_t)lane * 128u;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(rb + 16u * (uint32_t)(j ^ (lane & 7)), __float_as_uint(__uint_as_float(r[4 * j]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 1]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 2]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 3]) * scale));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // rows past T are clipped by the tensor map
        tma_reduce_add_3d(&tmDQ, box, h * HD + 32 * half, (kvb + t) * BQ + q * 32, b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(qdo_empty(sl));
      }
      __syncwarp();
    };
    // LSE (log2 domain) and D of every query block this CTA visits, once:
    // [block][LSE x128 | D x128]; queries past T get LSE = +inf (P = 0).
    // eight blocks' loads in flight at a time: a loop with a runtime trip
    // count would wait out one global-load latency per block
    const long bh0 = ((long)b * H + h) * T;
    for (int blk0 = 0; blk0 < nblk; blk0 += 8) {
      float vals[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int qq = (kvb + blk0 + u) * BQ + (tid & 127);
        const bool in = blk0 + u < nblk && qq < T;
        vals[u] = in ? (tid < 128 ? lse[bh0 + qq] * LOG2E_F : dvec[bh0 + qq]) : (tid < 128 ? INFINITY : 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (blk0 + u < nblk) sLD[(blk0 + u) * 256 + tid] = vals[u];
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    for (int t = 0; t < nblk; ++t) {
      const int q0 = (kvb + t) * BQ;
      const float* ld = sLD + t * 256;
      // masking only on the diagonal block, past T, or for keys past T
      const bool need_mask = (t == 0) || (q0 + BQ > T) || (kv >= T);
      if (!mbar_wait_bounded(st_full, t & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      // this warp's S^T / dP^T columns in two batches: the second batch is in
      // flight while the first is processed, and TMEM is released as soon as
      // it has landed so block t+1's S^T/dP^T MMAs overlap the math below
      uint32_t s[2][32], dp[2][32];
      tmem_ld_32x32b_x32(tmem + lane_off + C_ST + 64 * half, s[0]);
      tmem_ld_32x32b_x32(tmem + lane_off + C_DPT + 64 * half, dp[0]);
      tmem_ld_wait();
      tmem_ld_32x32b_x32(tmem + lane_off + C_ST + 64 * half + 32, s[1]);
      tmem_ld_32x32b_x32(tmem + lane_off + C_DPT + 64 * half + 32, dp[1]);
      uint32_t ppk[32], dpk[32];
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        if (sub == 1) {
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(st_free);
        }
        const int c0 = 64 * half + 32 * sub;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          // broadcast reads: every lane needs the same four columns
          const float4 l4 = *reinterpret_cast<const float4*>(ld + c0 + i);
          const float4 d4 = *reinterpret_cast<const float4*>(ld + 128 + c0 + i);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
          float pv[4], dv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float p = ex2(fmaf(__uint_as_float(s[sub][i + u]), scale_log2, -lv[u]));
            if (need_mask) {
              const int qq = q0 + c0 + i + u;
              if (qq < kv || qq >= T || kv >= T) p = 0.f;
            }
            pv[u] = p;
            dv[u] = p * (__uint_as_float(dp[sub][i + u]) - dd[u]);
          }
          ppk[sub * 16 + i / 2] = pack_bf16x2(pv[0], pv[1]);
          ppk[sub * 16 + i / 2 + 1] = pack_bf16x2(pv[2], pv[3]);
          dpk[sub * 16 + i / 2] = pack_bf16x2(dv[0], dv[1]);
          dpk[sub * 16 + i / 2 + 1] = pack_bf16x2(dv[2], dv[3]);
        }
      }
      // block t-1's dV/dK/dQ MMAs read P/dS: they must be done before the
      // buffers are overwritten (and before dQ(t-1) is drained below)
      if (t >= 1 && !mbar_wait_bounded(mma2_done, (t - 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      const uint32_t prow = base + BS_P + half * TILE + (uint32_t)row * 128u;
      const uint32_t drow = base + BS_DS + half * TILE + (uint32_t)row * 128u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t off = 16u * (uint32_t)(c ^ (row & 7));
        st_shared_v4(prow + off, ppk[4 * c], ppk[4 * c + 1], ppk[4 * c + 2], ppk[4 * c + 3]);
        st_shared_v4(drow + off, dpk[4 * c], dpk[4 * c + 1], dpk[4 * c + 2], dpk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ps_full);
      // dQ of block t-1 sits in the other TMEM buffer; reducing it into global
      // memory only after the release keeps these reductions off the MMA path.
      // Block t+1's dQ MMAs reuse that buffer only after this thread's next
      // ps_full arrival, which follows the completed loads below.
      if (t >= 1) drain_dq(t - 1);
    }
    if (ok && mbar_wait_bounded(mma2_done, (nblk - 1) & 1, abort_flag, err)) {
      tc_fence_after();
      drain_dq(nblk - 1);
      if (lane == 0) bulk_wait_all();
      uint32_t rk[32], rv[32];
      tmem_ld_32x32b_x32(tmem + lane_off + C_DK + 32 * half, rk);
      tmem_ld_32x32b_x32(tmem + lane_off + C_DV + 32 * half, rv);
      tmem_ld_wait();
      // dK and dV (this thread's row, 32 of the 64 columns) go to the K and V
      // tiles' shared memory (no MMA reads them any more) in the 128-byte
      // swizzle, and leave as two TMA stores (rows past T are clipped)
      const uint32_t krow = base + BS_K + (uint32_t)row * 128u, vrow = base + BS_V + (uint32_t)row * 128u;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int o = 8 * c;
        const uint32_t off = 16u * (uint32_t)((4 * half + c) ^ (row & 7));
        st_shared_v4(krow + off, pack_bf16x2(__uint_as_float(rk[o]) * scale, __uint_as_float(rk[o + 1]) * scale),
                     pack_bf16x2(__uint_as_float(rk[o + 2]) * scale, __uint_as_float(rk[o + 3]) * scale),
                     pack_bf16x2(__uint_as_float(rk[o + 4]) * scale, __uint_as_float(rk[o + 5]) * scale),
                     pack_bf16x2(__uint_as_float(rk[o + 6]) * scale, __uint_as_float(rk[o + 7]) * scale));
        st_shared_v4(vrow + off, pack_bf16x2(__uint_as_float(rv[o]), __uint_as_float(rv[o + 1])),
                     pack_bf16x2(__uint_as_float(rv[o + 2]), __uint_as_float(rv[o + 3])),
                     pack_bf16x2(__uint_as_float(rv[o + 4]), __uint_as_float(rv[o + 5])),
                     pack_bf16x2(__uint_as_float(rv[o + 6]), __uint_as_float(rv[o + 7])));
      }
      fence_proxy_async_smem();
      mbar_arrive(tail_bar);
      if (mbar_wait_bounded(tail_bar, 0, abort_flag, err) && warp == 2 && lane == 0) {
        tma_store_3d(&tmDQKV, base + BS_K, d + h * HD, kv0, b);
        tma_store_3d(&tmDQKV, base + BS_V, 2 * d + h * HD, kv0, b);
        bulk_commit();
        bulk_wait_all();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------ backward, persistent --
// Persistent over work items (128-key block, batch, head), longest first, in
// snake order over rounds.  Sixteen warps in four warpgroups with their own
// register budgets (setmaxnreg):
//   WG0  warp 0 TMA (K/V per item, double-buffered; Q/dO per query block),
//        warp 1 TMEM allocation and MMA issue, warps 2-3 idle      (80 regs)
//   WG1, WG2  elementwise: P^T = exp(S^T - LSE), dS^T = P^T (dP^T - D) for
//        64 query columns each; P^T goes to tensor memory (the dV product
//        reads it there), dS^T to a shared tile                          (168)
//   WG3  LSE/D staging two query blocks ahead, the dQ drain (tensor memory
//        -> shared -> TMA reduce-add into the fp32 dQ accumulator) and the
//        dK/dV write-out at the end of an item                           (96)
// The MMA warp issues S^T, dP^T of the next query block (the next item's
// first at an item's last) as soon as the elementwise warps have loaded the
// current ones, ahead of the current block's dV, dK, dQ products, so the
// elementwise work of one block overlaps the tensor-core work of the other.  Tensor memory: S^T 0-127, dP^T
// 128-255, P^T 256-319 (bf16 pairs), dV 320-383, dK 384-447, dQ 448-511.
namespace bw {
constexpr int QS = 3;  // Q/dO (and LSE/D) ring depth: loads run two query blocks ahead
constexpr int SM_KV = 0;                       // [item slot 2][K, V] tiles
constexpr int SM_QR = SM_KV + 4 * TILE;        // [QS] Q tiles
constexpr int SM_DOR = SM_QR + QS * TILE;      // [QS] dO tiles
constexpr int SM_DS = SM_DOR + QS * TILE;      // [2 halves] dS^T tile
constexpr int SM_DQ = SM_DS + 2 * TILE;        // [4 warps] 32 x 32 fp32 staging boxes
constexpr int SM_LD = SM_DQ + 4 * 4096;        // [QS][-LSE x128 | -D x128] floats
constexpr int SM_TILES = SM_LD + QS * 256 * 4;
// kv_full[2], kv_empty[2], qdo_full[QS], qdo_empty[QS], ld_full[QS], ld_empty[QS],
// st_full, st_free, ps_full, pt_free, ds_free, (spare), dq_full, dq_free,
// dkdv_full, dkdv_free, epi_stage, drain
constexpr int NUM_BARS = 4 + 4 * QS + 12;
constexpr int SMEM = SM_TILES + 1024 + NUM_BARS * 8 + 16;
static_assert(SMEM <= 232448, "backward shared memory");
constexpr int THREADS = 512;
constexpr uint32_t C_ST = 0, C_DPT = 128, C_PT = 256, C_DV = 320, C_DK = 384, C_DQ = 448;
// Register budgets per warpgroup after setmaxnreg; with 128 per thread at
// launch the block owns 512 x 128 = 65536 and the split below uses
// 128 x 80 + 256 x 168 + 128 x 96 = 65536 of them (the elementwise warps
// hold the most live values; 160 / 112 measured 1 % slower).
constexpr int LAUNCH_REGS = 128, REGS_CTRL = 80, REGS_ELEM = 168, REGS_DRAIN = 96;
static_assert(128 * REGS_CTRL + 256 * REGS_ELEM + 128 * REGS_DRAIN <= THREADS * LAUNCH_REGS, "register split");
}  // namespace bw

__global__ void __launch_bounds__(bw::THREADS, 1)
    attn_bwd_tc2_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDQKV,
                        const float* lse, const float* dvec, int T, int H, int n_items,
                        float scale, float scale_log2, int det, int* err) {
  // (local names shadow the one-CTA-per-block backward's constants above)
  constexpr int QS = bw::QS, SM_KV = bw::SM_KV, SM_QR = bw::SM_QR, SM_DOR = bw::SM_DOR, SM_DS = bw::SM_DS;
  constexpr int SM_DQ = bw::SM_DQ, SM_LD = bw::SM_LD, SM_TILES = bw::SM_TILES, NUM_BARS = bw::NUM_BARS;
  constexpr uint32_t C_ST = bw::C_ST, C_DPT = bw::C_DPT, C_PT = bw::C_PT, C_DV = bw::C_DV, C_DK = bw::C_DK,
                     C_DQ = bw::C_DQ;
  constexpr int REGS_CTRL = bw::REGS_CTRL, REGS_ELEM = bw::REGS_ELEM, REGS_DRAIN = bw::REGS_DRAIN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  float* sLD = reinterpret_cast<float*>(base_ptr + SM_LD);
  const uint32_t bars = base + SM_TILES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + SM_TILES + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto kv_full = [&](int s) { return bars + 8u * s; };
  auto kv_empty = [&](int s) { return bars + 8u * (2 + s); };
  auto qdo_full = [&](int r) { return bars + 8u * (4 + r); };
  auto qdo_empty = [&](int r) { return bars + 8u * (4 + QS + r); };
  auto ld_full = [&](int r) { return bars + 8u * (4 + 2 * QS + r); };
  auto ld_empty = [&](int r) { return bars + 8u * (4 + 3 * QS + r); };
  const uint32_t b0 = bars + 8u * (4 + 4 * QS);
  const uint32_t st_full = b0, st_free = b0 + 8, ps_full = b0 + 16, pt_free = b0 + 24;
  auto ds_free = [&](int i) { return b0 + 32u + 8u * i; };
  const uint32_t dq_full = b0 + 48, dq_free = b0 + 56, dkdv_full = b0 + 64, dkdv_free = b0 + 72;
  const uint32_t epi_stage = b0 + 80, drain_bar = b0 + 88;
  auto kv_tile = [&](int slot) { return base + SM_KV + (uint32_t)(2 * slot) * TILE; };  // K; V follows

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (T + BQ - 1) / BQ;
  const int BH = n_items / nqb;
  const int d = H * HD;
  // item w -> (key block, batch, head): low key blocks (most query blocks) first
  auto item = [&](int w, int& kb, int& b, int& h) {
    kb = w / BH;
    const int bh = w % BH;
    b = bh / H;
    h = bh % H;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 2);  // the item's last MMAs and the dK/dV store
    }
    mbar_init(ds_free(0), 1);
    for (int r = 0; r < QS; ++r) {
      mbar_init(qdo_full(r), 1);
      mbar_init(qdo_empty(r), 1);
      mbar_init(ld_full(r), 4);
      mbar_init(ld_empty(r), 8);
    }
    mbar_init(st_full, 1);
    mbar_init(st_free, 8);
    mbar_init(ps_full, 8);
    mbar_init(pt_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(dkdv_full, 1);
    mbar_init(dkdv_free, 4);
    mbar_init(epi_stage, 4);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmQKV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmDQ);
    tma_prefetch_desc(&tmDQKV);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_start();
  const int wg = warp >> 2;

  if (wg == 0) {
    reg_dealloc<REGS_CTRL>();
    if (warp == 0 && lane == 0) {
      // ----------------------------------------------------------- TMA ----
      bool ok = true;
      int it = 0, gq = 0, kv_issued = 0, q_issued = 0;
      for (int k = 0; ok; ++k, ++it) {
        const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
        if (w >= n_items) break;
        int kb, b, h;
        item(w, kb, b, h);
        const int nblk = nqb - kb, slot = it & 1;
        if (it >= 2 && !mbar_wait_bounded(kv_empty(slot), ((it - 2) >> 1) & 1, abort_flag, err)) { ok = false; break; }
        mbar_arrive_expect_tx(kv_full(slot), 2 * TILE);
        tma_load_3d(kv_tile(slot), &tmQKV, kv_full(slot), d + h * HD, kb * BKV, b);
        tma_load_3d(kv_tile(slot) + TILE, &tmQKV, kv_full(slot), 2 * d + h * HD, kb * BKV, b);
        ++kv_issued;
        for (int t = 0; t < nblk; ++t) {
          const int g = gq + t, r = g % QS;
          if (g >= QS && !mbar_wait_bounded(qdo_empty(r), ((g - QS) / QS) & 1, abort_flag, err)) { ok = false; break; }
          const int q0 = (kb + t) * BQ;
          mbar_arrive_expect_tx(qdo_full(r), 2 * TILE);
          tma_load_3d(base + SM_QR + r * TILE, &tmQKV, qdo_full(r), h * HD, q0, b);
          tma_load_3d(base + SM_DOR + r * TILE, &tmDO, qdo_full(r), h * HD, q0, b);
          ++q_issued;
        }
        gq += nblk;
      }
      if (!ok) {
        for (int i = kv_issued - 2 < 0 ? 0 : kv_issued - 2; i < kv_issued; ++i)
          mbar_drain_bounded(kv_full(i & 1), (i >> 1) & 1);
        for (int i = q_issued - QS < 0 ? 0 : q_issued - QS; i < q_issued; ++i)
          mbar_drain_bounded(qdo_full(i % QS), (i / QS) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      // ----------------------------------------------------------- MMA ----
      bool ok = true, issued_any = false;
      // S^T = K Q^T and dP^T = V dO^T of global query block g with the K / V
      // tiles at kt, vt
      auto issue_sdp = [&](int g, uint32_t kt, uint32_t vt) -> bool {
          const int r = g % QS;
          if (!mbar_wait_bounded(qdo_full(r), (g / QS) & 1, abort_flag, err)) return false;
          if (g >= 1 && !mbar_wait_bounded(st_free, (g - 1) & 1, abort_flag, err)) return false;
          tc_fence_after();
          const uint32_t qt = base + SM_QR + r * TILE, ot = base + SM_DOR + r * TILE;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc_mma_bf16(tmem + C_ST, sdesc(kt + kk * 32, 16, 1024), sdesc(qt + kk * 32, 16, 1024), IDESC_S,
                        kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc_mma_bf16(tmem + C_DPT, sdesc(vt + kk * 32, 16, 1024), sdesc(ot + kk * 32, 16, 1024), IDESC_S,
                        kk > 0 ? 1u : 0u);
          tc_commit(st_full);
          issued_any = true;
          return true;
      };
      int it = 0, gq = 0;
      int w = snake_item(0, (int)blockIdx.x, (int)gridDim.x);
      // the first item's K / V, and its first block's S^T, dP^T
      if (w < n_items) {
        ok = mbar_wait_bounded(kv_full(0), 0, abort_flag, err) && issue_sdp(0, kv_tile(0), kv_tile(0) + TILE);
      }
      for (int k = 0; ok && w < n_items; ++k, ++it) {
        int kb, b, h;
        item(w, kb, b, h);
        const int nblk = nqb - kb, slot = it & 1;
        const uint32_t kt = kv_tile(slot), vt = kt + TILE;
        const int wn = snake_item(k + 1, (int)blockIdx.x, (int)gridDim.x);
        for (int t = 0; t < nblk; ++t) {
          const int g = gq + t, r = g % QS;
          // the next block's S^T, dP^T ahead of this block's products; at the
          // item's last block that is the next item's first block, so the
          // elementwise warps do not wait out this block's products there
          if (t + 1 < nblk) {
            if (!issue_sdp(g + 1, kt, vt)) { ok = false; break; }
          } else if (wn < n_items) {
            const uint32_t kn = kv_tile(slot ^ 1);
            if (!mbar_wait_bounded(kv_full(slot ^ 1), ((it + 1) >> 1) & 1, abort_flag, err) ||
                !issue_sdp(g + 1, kn, kn + TILE)) { ok = false; break; }
          }
          if (!mbar_wait_bounded(ps_full, g & 1, abort_flag, err)) { ok = false; break; }
          // the previous item's dK / dV have been read out of tensor memory
          if (t == 0 && it >= 1 && !mbar_wait_bounded(dkdv_free, (it - 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qt = base + SM_QR + r * TILE, ot = base + SM_DOR + r * TILE;
          const uint32_t ds = base + SM_DS;
          // dV += P^T dO (P^T from tensor memory)
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            tc_mma_bf16_ts(tmem + C_DV, tmem + C_PT + 8u * kk, sdesc(ot + kk * 2048, 8192, 1024), IDESC_O,
                           (t > 0 || kk > 0) ? 1u : 0u);
          tc_commit(pt_free);
          // dK += dS^T Q
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            tc_mma_bf16(tmem + C_DK, sdesc(ds + (kk >> 2) * TILE + (kk & 3) * 32, 16, 1024),
                        sdesc(qt + kk * 2048, 8192, 1024), IDESC_O, (t > 0 || kk > 0) ? 1u : 0u);
          // dQ = dS K into the single dQ buffer, once its previous block is drained
          if (g >= 1 && !mbar_wait_bounded(dq_free, (g - 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            tc_mma_bf16(tmem + C_DQ, sdesc(ds + kk * 2048, TILE, 1024), sdesc(kt + kk * 2048, 8192, 1024), IDESC_DQ,
                        kk > 0 ? 1u : 0u);
          tc_commit(dq_full);
          tc_commit(ds_free(0));
          tc_commit(qdo_empty(r));
        }
        if (!ok) break;
        tc_commit(dkdv_full);
        tc_commit(kv_empty(slot));
        gq += nblk;
        w = wn;
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_drain_bounded(drain_bar, 0);
      }
    }
  } else if (wg <= 2) {
    reg_alloc<REGS_ELEM>();
    // --------------------------------------------------------- elementwise ----
    const int q = warp & 3;          // TMEM lanes [32q, 32q+32): key rows
    const int half = wg - 1;         // query columns [64 half, 64 half + 64)
    const int row = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    bool ok = true;
    int gq = 0;
    for (int k = 0; ok; ++k) {
      const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
      if (w >= n_items) break;
      int kb, b, h;
      item(w, kb, b, h);
      const int nblk = nqb - kb;
      const int kv = kb * BKV + row;
      for (int t = 0; t < nblk; ++t) {
        const int g = gq + t, r = g % QS;
        const int q0 = (kb + t) * BQ;
        if (!mbar_wait_bounded(ld_full(r), (g / QS) & 1, abort_flag, err)) { ok = false; break; }
        if (!mbar_wait_bounded(st_full, g & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        // masking only on the diagonal block, past T, or for keys past T
        const bool need_mask = (t == 0) || (q0 + BQ > T) || (kv >= T);
        const float* ld = sLD + r * 256;  // -LSE, -D
        uint32_t pp[32], pd[32];
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        // the two 32-column halves one after the other (fewer live
        // registers); S^T / dP^T are released once both halves are loaded
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          uint32_t sv[1][32], dp[1][32];
          tmem_ld_32x32b_x32(tmem + lane_off + C_ST + 64 * half + 32 * sub, sv[0]);
          tmem_ld_32x32b_x32(tmem + lane_off + C_DPT + 64 * half + 32 * sub, dp[0]);
          tmem_ld_wait();
          if (sub == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(st_free);
          }
          const int c0 = 64 * half + 32 * sub;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            // broadcast reads: every lane needs the same four columns
            const float4 l4 = *reinterpret_cast<const float4*>(ld + c0 + i);
            const float4 d4 = *reinterpret_cast<const float4*>(ld + 128 + c0 + i);
            // two columns per packed fp32x2 operation
            const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sv[0][i]), __uint_as_float(sv[0][i + 1])),
                                          sc2, make_float2(l4.x, l4.y));
            const float2 x23 = __ffma2_rn(
                make_float2(__uint_as_float(sv[0][i + 2]), __uint_as_float(sv[0][i + 3])), sc2,
                make_float2(l4.z, l4.w));
            const float pv[4] = {ex2(x01.x), ex2(x01.y), ex2(x23.x), ex2(x23.y)};
            const float2 e01 = __fadd2_rn(make_float2(__uint_as_float(dp[0][i]), __uint_as_float(dp[0][i + 1])),
                                          make_float2(d4.x, d4.y));
            const float2 e23 = __fadd2_rn(
                make_float2(__uint_as_float(dp[0][i + 2]), __uint_as_float(dp[0][i + 3])),
                make_float2(d4.z, d4.w));
            const float2 g01 = __fmul2_rn(make_float2(pv[0], pv[1]), e01);
            const float2 g23 = __fmul2_rn(make_float2(pv[2], pv[3]), e23);
            pp[sub * 16 + i / 2] = pack_bf16x2(pv[0], pv[1]);
            pp[sub * 16 + i / 2 + 1] = pack_bf16x2(pv[2], pv[3]);
            pd[sub * 16 + i / 2] = pack_bf16x2(g01.x, g01.y);
            pd[sub * 16 + i / 2 + 1] = pack_bf16x2(g23.x, g23.y);
          }
        }
        if (need_mask) {
          // the causal and ragged masks: the packed P and dS words of masked
          // columns (two columns a word) cleared after the fact, so that the
          // unrolled loop above carries no mask code.  Column c of this
          // half (query q0 + 64 half + c) stays iff lo <= c < hi.
          const int lo = kv - (q0 + 64 * half);
          const int hi = kv < T ? T - (q0 + 64 * half) : lo;
#pragma unroll
          for (int w = 0; w < 32; ++w) {
            const uint32_t m = (2 * w >= lo && 2 * w < hi ? 0x0000ffffu : 0u) |
                               (2 * w + 1 >= lo && 2 * w + 1 < hi ? 0xffff0000u : 0u);
            pp[w] &= m;
            pd[w] &= m;
          }
        }
        // every lane has read this block's LSE / D
        __syncwarp();
        if (lane == 0) mbar_arrive(ld_empty(r));
        // dV of the previous block has read P^T, its dK and dQ have read dS^T
        // (they are issued right after this warp's previous release, and this
        // block's arithmetic above is longer than they take)
        if (g >= 1 && !mbar_wait_bounded(pt_free, (g - 1) & 1, abort_flag, err)) { ok = false; break; }
        if (g >= 1 && !mbar_wait_bounded(ds_free(0), (g - 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        tmem_st_32x32b_x32(tmem + lane_off + C_PT + 32 * half, pp);
        const uint32_t drow = base + SM_DS + half * TILE + (uint32_t)row * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(drow + 16u * (uint32_t)(c ^ (row & 7)), pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ps_full);
      }
      gq += nblk;
    }
  } else {
    reg_dealloc<REGS_DRAIN>();
    // ---------------------------------------- LSE/D staging, dQ, dK / dV ----
    const int q = warp & 3;  // TMEM lanes [32q, 32q+32): query rows of dQ, key rows of dK / dV
    const int tid = threadIdx.x - 384;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t box = base + SM_DQ + (uint32_t)q * 4096u;
    bool ok = true;
    // -LSE (log2 domain) and -D of a query block into its ring slot (queries
    // past T: -LSE = -inf, -D = 0), negated so the elementwise warps need one
    // fused multiply-add and one add per pair.  Staged two query blocks ahead
    // along this CTA's sequence of (item, query block): the global loads of
    // block g + 2 are issued before block g's dQ drain and written to the ring
    // after it, so their latency overlaps the drain instead of preceding it.
    int ks = 0, ts = 0, kbs = 0, bs = 0, hs = 0, nbs = 0;  // the staging cursor
    bool have = false;
    auto cursor_item = [&](int kk) {
      const int w = snake_item(kk, (int)blockIdx.x, (int)gridDim.x);
      have = w < n_items;
      if (have) {
        item(w, kbs, bs, hs);
        nbs = nqb - kbs;
        ks = kk;
        ts = 0;
      }
    };
    auto cursor_next = [&]() {
      if (++ts >= nbs) cursor_item(ks + 1);
    };
    auto stage_load = [&](float& lv, float& dv) {
      const int qq = (kbs + ts) * BQ + tid;
      const long bh0 = ((long)bs * H + hs) * T;
      lv = qq < T ? lse[bh0 + qq] : 0.f;
      dv = qq < T ? dvec[bh0 + qq] : 0.f;
    };
    // the cursor's block, number g of the sequence, into ring slot g % QS
    auto stage_store = [&](int g, float lv, float dv) -> bool {
      const int r = g % QS;
      if (g >= QS && !mbar_wait_bounded(ld_empty(r), ((g - QS) / QS) & 1, abort_flag, err)) return false;
      const int qq = (kbs + ts) * BQ + tid;
      sLD[r * 256 + tid] = qq < T ? -lv * LOG2E_F : -INFINITY;
      sLD[r * 256 + 128 + tid] = qq < T ? -dv : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(ld_full(r));
      return true;
    };
    int staged = 0;  // query blocks staged so far
    cursor_item(0);
    for (int i = 0; i < 2 && have && ok; ++i) {
      float lv, dv;
      stage_load(lv, dv);
      ok = stage_store(staged, lv, dv);
      ++staged;
      cursor_next();
    }
    int gq = 0, it = 0;
    for (int k = 0; ok; ++k, ++it) {
      const int w = snake_item(k, (int)blockIdx.x, (int)gridDim.x);
      if (w >= n_items) break;
      int kb, b, h;
      item(w, kb, b, h);
      const int nblk = nqb - kb, slot = it & 1;
      for (int t = 0; t < nblk; ++t) {
        const int g = gq + t;
        // block g + 2's LSE / D: loaded now, written after this block's dQ drain
        const bool pend = have;
        float lv = 0.f, dv = 0.f;
        if (pend) stage_load(lv, dv);
        // dQ of block g: tensor memory -> registers (the buffer is then free
        // for the next block's dQ) -> two 32 x 32 fp32 boxes -> TMA reduce-add
        // (bulk reductions into L2; per-lane vector reductions measured slower)
        if (!mbar_wait_bounded(dq_full, g & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        uint32_t dq[2][32];
        tmem_ld_32x32b_x32(tmem + lane_off + C_DQ, dq[0]);
        tmem_ld_32x32b_x32(tmem + lane_off + C_DQ + 32, dq[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);
        const int q0 = (kb + t) * BQ;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          // this warp's box was last read by the previous reduce
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
          const uint32_t rb = box + (uint32_t)lane * 128u;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(rb + 16u * (uint32_t)(j ^ (lane & 7)), __float_as_uint(__uint_as_float(dq[c][4 * j]) * scale),
                         __float_as_uint(__uint_as_float(dq[c][4 * j + 1]) * scale),
                         __float_as_uint(__uint_as_float(dq[c][4 * j + 2]) * scale),
                         __float_as_uint(__uint_as_float(dq[c][4 * j + 3]) * scale));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past T are clipped by the tensor map.  Deterministic mode:
            // the tile goes to the key block's own slice of the partial buffer
            // (z = key block * batch + batch index), summed later in order
            if (det)
              tma_store_3d(&tmDQ, box, h * HD + 32 * c, q0 + q * 32, kb * (BH / H) + b);
            else
              tma_reduce_add_3d(&tmDQ, box, h * HD + 32 * c, q0 + q * 32, b);
            bulk_commit();
          }
        }
        if (pend) {
          if (!stage_store(staged, lv, dv)) { ok = false; break; }
          ++staged;
          cursor_next();
        }
      }
      if (!ok) break;
      // ---- dK (scaled) and dV of the item, bf16, through its K / V tiles
      if (!mbar_wait_bounded(dkdv_full, it & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      const int row = q * 32 + lane;
      const uint32_t kt = kv_tile(slot), vt = kt + TILE;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        uint32_t o[2][32];
        tmem_ld_32x32b_x32(tmem + lane_off + (which ? C_DV : C_DK), o[0]);
        tmem_ld_32x32b_x32(tmem + lane_off + (which ? C_DV : C_DK) + 32, o[1]);
        tmem_ld_wait();
        if (which == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dkdv_free);
        }
        const float sc = which ? 1.f : scale;
        const uint32_t orow = (which ? vt : kt) + (uint32_t)row * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t* oc = &o[c >> 2][(c & 3) * 8];
          st_shared_v4(orow + 16u * (uint32_t)(c ^ (row & 7)),
                       pack_bf16x2(__uint_as_float(oc[0]) * sc, __uint_as_float(oc[1]) * sc),
                       pack_bf16x2(__uint_as_float(oc[2]) * sc, __uint_as_float(oc[3]) * sc),
                       pack_bf16x2(__uint_as_float(oc[4]) * sc, __uint_as_float(oc[5]) * sc),
                       pack_bf16x2(__uint_as_float(oc[6]) * sc, __uint_as_float(oc[7]) * sc));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_stage);
      if (!mbar_wait_bounded(epi_stage, it & 1, abort_flag, err)) { ok = false; break; }
      if (warp == 12 && lane == 0) {
        // rows past T are clipped by the tensor map
        tma_store_3d(&tmDQKV, kt, d + h * HD, kb * BKV, b);
        tma_store_3d(&tmDQKV, vt, 2 * d + h * HD, kb * BKV, b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(kv_empty(slot));
      }
      __syncwarp();
      gq += nblk;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

int attn_tc_set_wait_limit(unsigned long long ns) { return set_unit_wait_limit(ns); }

int attn_bwd_tc(const void* qkv, const void* dout, const float* lse, const float* dvec, void* dqkv, float* dq_acc,
                int B, int T, int H, cudaStream_t st, float* dq_part) {
  if (B <= 0 || T <= 0) return GPT2_OK;
  if ((T + BQ - 1) / BQ > BS_MAX_QBLOCKS) return GPT2_ERR_UNSUPPORTED_SHAPE;
  const uint64_t d = (uint64_t)H * HD;
  const uint64_t nqb = (uint64_t)((T + BQ - 1) / BQ);
  CUtensorMap tq, tdo;
  const uint64_t dq[3] = {3 * d, (uint64_t)T, (uint64_t)B};
  const uint64_t sq[2] = {3 * d * 2, (uint64_t)T * 3 * d * 2};
  const uint64_t dd[3] = {d, (uint64_t)T, (uint64_t)B};
  const uint64_t sd[2] = {d * 2, (uint64_t)T * d * 2};
  CUtensorMap tdq, tdqkv;
  const uint64_t sdq[2] = {d * 4, (uint64_t)T * d * 4};
  // deterministic mode: [key block][batch] slices of [T, d] fp32
  const uint64_t dpart[3] = {d, (uint64_t)T, nqb * (uint64_t)B};
  if (!tmap_3d(&tq, qkv, dq, sq) || !tmap_3d(&tdo, dout, dd, sd) ||
      !tmap_3d(&tdq, dq_part ? dq_part : dq_acc, dq_part ? dpart : dd, sdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 32,
               32) ||
      !tmap_3d(&tdqkv, dqkv, dq, sq))
    return GPT2_ERR_CUDA;
  // The persistent kernel, if its launch register count is the one its
  // register split is computed for (otherwise a setmaxnreg.inc could wait for
  // registers the block does not own): checked once on the host.
  static int v2 = -1;
  if (v2 < 0) {
    const char* e = getenv("GPT2_ATTN_BWD_TC");
    cudaFuncAttributes fa;
    v2 = (e && e[0] == '1') ? 0
         : (cudaFuncGetAttributes(&fa, attn_bwd_tc2_kernel) == cudaSuccess && fa.numRegs == bw::LAUNCH_REGS) ? 1
                                                                                                             : 0;
    cudaGetLastError();
  }
  if (v2) {
    CUDA_TRY(once_per_device((const void*)attn_bwd_tc2_kernel, [](int) {
      return cudaFuncSetAttribute(attn_bwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bw::SMEM);
    }));
    const int n_items = ((T + BKV - 1) / BKV) * B * H;
    const int grid = n_items < num_sms() ? n_items : num_sms();
    CUDA_TRY(launch_k(attn_bwd_tc2_kernel, grid, bw::THREADS, bw::SMEM, st, tq, tdo, tdq, tdqkv, lse, dvec, T, H,
                      n_items, 0.125f, LOG2E_F / 8.f, dq_part ? 1 : 0, nullptr));
    LAUNCH_CHECK();
    return GPT2_OK;
  }
  if (dq_part) return GPT2_ERR_UNSUPPORTED_SHAPE;  // (a mode of the persistent kernel only)
  CUDA_TRY(once_per_device((const void*)attn_bwd_tc_kernel, [](int) {
    return cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM_BYTES);
  }));
  dim3 grid((T + BKV - 1) / BKV, B * H);
  CUDA_TRY(launch_k(attn_bwd_tc_kernel, grid, B_NUM_THREADS, B_SMEM_BYTES, st, tq, tdo, tdq, tdqkv, lse, dvec, T, H,
                                                                 0.125f, LOG2E_F / 8.f, nullptr));
  LAUNCH_CHECK();
  return GPT2_OK;
}

int attn_fwd_tc(const void* qkv, void* o, float* lse, int B, int T, int H, cudaStream_t st) {
  if (B <= 0 || T <= 0) return GPT2_OK;
  const uint64_t d = (uint64_t)H * HD;
  CUtensorMap tq, to;
  const uint64_t dq[3] = {3 * d, (uint64_t)T, (uint64_t)B};
  const uint64_t sq[2] = {3 * d * 2, (uint64_t)T * 3 * d * 2};
  const uint64_t dout[3] = {d, (uint64_t)T, (uint64_t)B};
  const uint64_t sout[2] = {d * 2, (uint64_t)T * d * 2};
  if (!tmap_3d(&tq, qkv, dq, sq) || !tmap_3d(&to, o, dout, sout)) return GPT2_ERR_CUDA;
  // The two-tile kernel, if its launch register count is the one its
  // register split is computed for (checked once on the host; "1" in
  // GPT2_ATTN_FWD_TC selects the one-tile kernel, for comparison).
  static int v2 = -1;
  if (v2 < 0) {
    const char* e = getenv("GPT2_ATTN_FWD_TC");
    cudaFuncAttributes fa;
    v2 = (e && e[0] == '1') ? 0
         : (cudaFuncGetAttributes(&fa, attn_fwd_tc2_kernel) == cudaSuccess && fa.numRegs == F2_LAUNCH_REGS) ? 1
                                                                                                           : 0;
    cudaGetLastError();
  }
  if (v2) {
    CUDA_TRY(once_per_device((const void*)attn_fwd_tc2_kernel, [](int) {
      return cudaFuncSetAttribute(attn_fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, F2_SMEM);
    }));
    const int nqb = (T + BQ - 1) / BQ;
    const int n_items = ((nqb + 1) / 2) * B * H;
    const int grid = n_items < num_sms() ? n_items : num_sms();
    CUDA_TRY(launch_k(attn_fwd_tc2_kernel, grid, F2_THREADS, F2_SMEM, st, tq, to, lse, T, H, n_items,
                      LOG2E_F / 8.f, nullptr));
    LAUNCH_CHECK();
    return GPT2_OK;
  }
  CUDA_TRY(once_per_device((const void*)attn_fwd_tc_kernel, [](int) {
    return cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  }));
  const int n_items = ((T + BQ - 1) / BQ) * B * H;
  const int grid = n_items < num_sms() ? n_items : num_sms();
  CUDA_TRY(launch_k(attn_fwd_tc_kernel, grid, NUM_THREADS, SMEM_BYTES, st,
      tq, to, lse, T, H, n_items, LOG2E_F / 8.f, nullptr));
  LAUNCH_CHECK();
  return GPT2_OK;
}
