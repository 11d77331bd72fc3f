// Host side of the tcgen05 GEMM: tensor maps, tile and split-K choice, the
// epilogue's store mode, and the launch of the kernel instantiation for the
// epilogue kind (the instantiations live in gemm_tc_pair.cu and
// gemm_tc_single.cu so that they compile in parallel).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "gemm_tc.cuh"

namespace tcg {
TCG_FOR_EACH_KIND(TCG_DECLARE, 256, true)
TCG_DECLARE(256, true, EPI_CE_FWD)
TCG_FOR_EACH_KIND(TCG_DECLARE, 256, false)
TCG_DECLARE(256, false, EPI_CE_FWD)
TCG_FOR_EACH_KIND(TCG_DECLARE, 128, false)
}  // namespace tcg

using namespace tcg;

namespace {

// out = beta*out + alpha * sum_s part[s]   (fixed order over s)
__global__ void splitk_reduce_kernel(const float* part, int splits, long mn,
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

// bf16 out = alpha * sum_s part[s]   (fixed order over s; mn a multiple of 4)
__global__ void splitk_reduce_bf16_kernel(const float* part, int splits, long mn,
                                          bf16* __restrict__ out, float alpha) {
  pdl_start();
  const long i = (blockIdx.x * (long)blockDim.x + threadIdx.x) * 4;
  if (i >= mn) return;
  float4 acc = reinterpret_cast<const float4*>(part + i)[0];
  for (int s = 1; s < splits; ++s) {
    const float4 t = reinterpret_cast<const float4*>(part + (long)s * mn + i)[0];
    acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
  }
  uint2 o;
  o.x = pack_bf16x2(alpha * acc.x, alpha * acc.y);
  o.y = pack_bf16x2(alpha * acc.z, alpha * acc.w);
  *reinterpret_cast<uint2*>(out + i) = o;
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

// [M, N] with pitch ldo in 32-row boxes, 128-byte swizzle (the layout the
// epilogue writes and reads): bf16 boxes of 64 columns, fp32 of 32.
bool make_out_tmap(CUtensorMap* tm, const void* base, int M, int N, long ldo, bool f32) {
  const uint64_t dims[2] = {(uint64_t)N, (uint64_t)M}, strides[1] = {(uint64_t)ldo * (f32 ? 4 : 2)};
  const uint32_t box[2] = {f32 ? 32u : 64u, 32};
  return encode_tmap(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2,
                     dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
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
//   + s * M * N * 8 bytes (partials written and read back) / HBM bandwidth
//   + (s > 3: the separate reduction launch; up to 3 splits are reduced
//      inside the kernel),
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
  const double reduce_us = 4.0;       // a reduction launch: its set-up and tail
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 16 && s <= kb / 4; ++s) {
    const long units = tiles * s;
    const long waves = (units + slots - 1) / slots;
    const double cost = (double)waves * ((double)kb / s) * kblock_us +
                        (s > 1 ? (double)s * M * N * 8.0 / bytes_per_us : 0.0) + (s > 3 ? reduce_us : 0.0);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

}  // namespace

// SMs of the current device (per device: a process may drive several)
int num_sms() {
  static int n[MAX_DEVICES] = {};
  const int dev = current_device();
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    n[dev] = v;
  }
  return n[dev];
}

int gemm_tc_pair_set_wait_limit(unsigned long long ns);
int gemm_tc_single_set_wait_limit(unsigned long long ns);
// the kernels live in the two instantiation units, each with its own limit
int gemm_tc_set_wait_limit(unsigned long long ns) {
  const int rc = gemm_tc_pair_set_wait_limit(ns);
  return rc ? rc : gemm_tc_single_set_wait_limit(ns);
}

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
  // With per-tile counters an fp32 output (beta 0 or 1) is split in order
  // inside the kernel: S - 1 partial slices, no separate reduction pass.
  const int tiles = ((g.M + (pair ? 2 * BM : BM) - 1) / (pair ? 2 * BM : BM)) * ((g.N + n_mma - 1) / n_mma);
  // (The last split reads the earlier partials one after another, so deeper
  // splits keep the separate reduction.)
  bool serial = splits > 1 && splits <= 3 && g.epi.kind == EPI_F32 && g.epi.split_cnt &&
                (g.epi.beta == 0.f || g.epi.beta == 1.f) &&
                (long)tiles * (pair ? 2 : 1) * NUM_EPI_WARPS <= g.epi.split_cnt_len;
  if (splits > 1) {
    // fp32 (weight-gradient) outputs, or a plain bf16 store: partial sums in
    // the workspace, then a fixed-order reduction
    if ((g.epi.kind != EPI_F32 && g.epi.kind != EPI_STORE) || g.N % 4 || g.epi.ldo != g.N)
      return GPT2_ERR_INVALID_ARG;
    size_t need = (size_t)(serial ? splits - 1 : splits) * g.M * g.N * sizeof(float);
    if (!ws || ws_bytes < need) splits = 1;
  }
  if (splits <= 1) serial = false;

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
  // the larger operand's tiles are the ones the concurrent units share
  p.n_fast = g.M > g.N ? 1 : 0;
  p.kb_total = kb_total;
  // instruction descriptor, kind::f16: D fp32 (bit 4), A and B bf16 (bits 7, 10),
  // operand majorness (bits 15, 16), N >> 3 at bit 17, M >> 4 at bit 24 (M = 256
  // for a CTA pair: 128 rows in each CTA).
  p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)g.a_mn << 15) | ((uint32_t)g.b_mn << 16) |
            ((uint32_t)(n_mma >> 3) << 17) | ((uint32_t)(p.tile_m >> 4) << 24);
  p.epi = g.epi;
  p.partial = (float*)ws;
  p.err = err;
  p.serial = serial ? 1 : 0;
  if (splits > 1 && !serial) {
    // raw partial sums: the reduction applies alpha and beta
    p.epi.kind = EPI_F32_PARTIAL;
    p.epi.alpha = 1.f;
  }

  // output path: TMA stores of 32-row boxes staged in shared memory
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
      // the optional column-sum partials are written as fp32 pairs
      if (p.epi.kind == EPI_DGELU && g.epi.colsum && (((uintptr_t)g.epi.colsum & 7) || (g.N & 1)))
        return GPT2_ERR_INVALID_ARG;
      // tmC2: the operand read per 64-column half (same [M, ldo] layout as the output)
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
      if (serial) {
        // tmC2: the partial slices [split][M][N] of splits 0 .. S-2
        const uint64_t dims[3] = {(uint64_t)g.N, (uint64_t)g.M, (uint64_t)(splits - 1)};
        const uint64_t strides[2] = {(uint64_t)g.N * 4, (uint64_t)g.M * g.N * 4};
        const uint32_t box[3] = {32, 32, 1};
        ok_c = ok_c && encode_tmap(&tc2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ws, 3, dims, strides, box,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
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
      return GPT2_ERR_INVALID_ARG;
  }
  if (!ok_c) return GPT2_ERR_CUDA;

  const int units = p.m_tiles * p.n_tiles * splits;
  const int ek = p.epi.kind == EPI_F32_PARTIAL ? EPI_F32 : p.epi.kind;
  int rc = GPT2_ERR_INVALID_ARG;
#define TCG_CASE(BN_, PAIR_, EK_) \
  case EK_:                      \
    rc = launch_tc<BN_, PAIR_, EK_>(ta, tb, tc, tc2, p, units, st); \
    break;
  if (pair) {
    switch (ek) {
      TCG_FOR_EACH_KIND(TCG_CASE, 256, true)
      TCG_CASE(256, true, EPI_CE_FWD)
    }
  } else if (bn == 256) {
    switch (ek) {
      TCG_FOR_EACH_KIND(TCG_CASE, 256, false)
      TCG_CASE(256, false, EPI_CE_FWD)
    }
  } else {
    switch (ek) {
      TCG_FOR_EACH_KIND(TCG_CASE, 128, false)
    }
  }
#undef TCG_CASE
  if (rc) return rc;
  if (splits > 1 && !serial) {
    long mn = (long)g.M * g.N;
    long threads = (mn + 3) / 4;
    if (g.epi.kind == EPI_STORE)
      CUDA_TRY(launch_k(splitk_reduce_bf16_kernel, (unsigned)((threads + 255) / 256), 256, 0, st,
                        (const float*)ws, splits, mn, (bf16*)g.epi.out, g.epi.alpha));
    else
      CUDA_TRY(launch_k(splitk_reduce_kernel, (unsigned)((threads + 255) / 256), 256, 0, st,
                        (const float*)ws, splits, mn, (float*)g.epi.out, g.epi.alpha, g.epi.beta));
    LAUNCH_CHECK();
  }
  return GPT2_OK;
}
