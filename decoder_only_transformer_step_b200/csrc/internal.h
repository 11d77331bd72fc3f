// Host-side interface between the library's compilation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

// Epilogue applied to each GEMM output element (row m, column n, fp32 acc).
// "act" is the activation type of the mode (bf16 or fp32).
enum EpiKind : int {
  EPI_STORE = 0,    // out(act)  = alpha * acc
  EPI_BIAS,         // out(act)  = acc + bias[n]
  EPI_BIAS_RESID,   // out(act)  = acc + bias[n] + resid[m,n]
  EPI_BIAS_GELU,    // u = acc + bias[n]: out(act) = gelu'(u), out2(act) = gelu(u)
  EPI_DGELU,        // out(act)  = acc * aux[m,n]  (aux = the saved gelu'(u)); optionally
                    //   colsum[m/32][n] = sum of out over rows 32 (m/32) .. 32 (m/32) + 31
  EPI_F32,          // out(fp32) = beta * out + alpha * acc
  EPI_F32_PARTIAL,  // partial[split][m,n] = acc (split-K, internal)
  EPI_ROWDOT,       // out(bf16) = acc; out2(fp32)[(m / seq * N/64 + n/64) * seq + m % seq] =
                    //   sum over the 64 columns of head n/64 of bf16(acc) * aux[m,n]
  EPI_CE_FWD,       // LM head with the cross-entropy's online log-sum-exp: per row m and
                    //   128-column part p (N % 128 == 0): ce_max[p*M+m] = max_n acc,
                    //   out(bf16)[m,n] = exp(acc - ce_max), ce_sum[p*M+m] = sum of those
                    //   (fp32), ce_zt[m] = acc[m, ce_tgt[m]] (fp32) when 0 <= ce_tgt[m] < N
};

struct EpiArgs {
  int kind;
  void* out;          // [M, ldo]
  void* out2;         // [M, ldo] (EPI_BIAS_GELU)
  const void* bias;   // [N] act
  const void* resid;  // [M, ldo] act
  const void* aux;    // [M, ldo] act
  long ldo;
  float alpha, beta;
  int seq;            // EPI_ROWDOT: rows per sequence
  float* colsum;      // EPI_DGELU, optional: [ceil(M/32), N] fp32 sums of the stored (bf16)
                      //   output over each 32-row group (the bias gradient's partials)
  int* split_cnt;     // EPI_F32 split along K, optional: zeroed per-tile counters that order
  int split_cnt_len;  //   the splits inside the kernel (no separate reduction pass)
  // EPI_CE_FWD
  float* ce_max;
  float* ce_sum;
  float* ce_zt;
  const int32_t* ce_tgt;
};

struct GemmArgs {
  int M, N, K;
  const void* A; int a_mn; long lda;
  const void* B; int b_mn; long ldb;
  EpiArgs epi;
};

// tcgen05 bf16 GEMM (sm_100a).  ws (may be NULL) holds split-K partials for
// EPI_F32.  bn: 0 auto / 128 / 256; splits: 0 auto.
int gemm_tc_bf16(const GemmArgs& g, void* ws, size_t ws_bytes, int bn, int splits, int* err,
                 cudaStream_t st);
// Workspace bytes the automatic split-K choice wants for this problem.
size_t gemm_tc_split_bytes(int M, int N, int K);

// fp32 CUDA-core GEMM for the correctness mode.
int gemm_simt_f32(const GemmArgs& g, cudaStream_t st);

int num_sms();

// Limit (ns) of the pipeline waits of the tcgen05 GEMM / attention kernels on
// the current device.
int gemm_tc_set_wait_limit(unsigned long long ns);
int attn_tc_set_wait_limit(unsigned long long ns);

// tcgen05 causal attention forward / backward, head_dim 64 (bf16).  The
// backward expects dvec = rowsum(dO * O) and a zeroed fp32 dq_acc; it writes dK,
// dV into dqkv and reduces scale * dQ into dq_acc.
int attn_fwd_tc(const void* qkv, void* o, float* lse, int B, int T, int H, cudaStream_t st);
int attn_bwd_tc(const void* qkv, const void* dout, const float* lse, const float* dvec, void* dqkv, float* dq_acc,
                int B, int T, int H, cudaStream_t st, float* dq_part = nullptr);

// ---- attention ----------------------------------------------------------
// qkv [B*T, 3*H*hd] (act), o [B*T, H*hd] (act), lse [B,H,T] fp32.
int attn_fwd_bf16(const void* qkv, void* o, float* lse, int B, int T, int H, int hd,
                  cudaStream_t st);
int attn_fwd_f32(const float* qkv, float* o, float* lse, int B, int T, int H, int hd,
                 cudaStream_t st);
// dq_acc: fp32 [B*T, H*hd] scratch; dvec: fp32 [B,H,T] scratch.  With
// dvec_ready the caller has already written dvec = rowsum(dO * O) (head_dim 64:
// the EPI_ROWDOT epilogue of the GEMM that produced dO) and zeroed dq_acc; the
// call leaves dq_acc zeroed again for the next layer.
// With dq_part (fp32 [ceil(T/128)][B*T][H*hd], head_dim 64, T <= 4096) every
// key block's dQ tile is stored in its own slice and the slices are added in
// key-block order: bitwise repeatable (dq_acc is then not used).
int attn_bwd_bf16(const void* qkv, const void* o, const float* lse, const void* dout, void* dqkv,
                  float* dq_acc, float* dvec, int B, int T, int H, int hd, cudaStream_t st, int dvec_ready = 0,
                  float* dq_part = nullptr);
int attn_bwd_f32(const float* qkv, const float* o, const float* lse, const float* dout,
                 float* dqkv, float* dvec, int B, int T, int H, int hd, cudaStream_t st);

// ---- elementwise / reductions (templated on bf16 = 0 / fp32 = 1) -------
int embed_fwd(int f32, const int32_t* tok, const void* wte, const void* wpe, void* x, int M, int T,
              int d, int vocab_real, int* err, cudaStream_t st);
int layernorm_fwd(int f32, const void* x, const void* g, const void* b, void* y, float* mean,
                  float* rstd, int M, int d, cudaStream_t st);
// dres = (dres_init ? 0 : dres) + LN'(dy); writes per-block partials of
// dgamma, dbeta into part [nblk, 2, d] and, if part_res is not NULL, the
// column sums of the new dres into part_res [nblk, d]; returns nblk.
int layernorm_bwd(int f32, const void* dy, const void* x, const float* mean, const float* rstd,
                  const void* g, void* dres, int dres_init, float* part, float* part_res, int* nblk, int M,
                  int d, cudaStream_t st);
// rows of those partial buffers (floats: rows * 2d and rows * d)
size_t layernorm_bwd_part_rows(int M);
size_t layernorm_bwd_part_floats(int M, int d);
// grad[j] = beta*grad[j] + sum_b part[b, j]  for j < n  (part row pitch n)
int reduce_rows_f32(const float* part, int nrows, int n, float* grad, float beta, cudaStream_t st);
// Many such reductions in one launch (same per-column summation order).
struct ReduceJob {
  const float* part;
  float* grad;
  int nrows, n;
};
constexpr int MAX_REDUCE_JOBS = 96;
int reduce_rows_batch(const ReduceJob* jobs, int njobs, float beta, cudaStream_t st);
// per-block column sums of x [M, N] (act) into part [nblk, N]
int colsum_partial(int f32, const void* x, int M, int N, float* part, int* nblk, cudaStream_t st);
size_t colsum_part_floats(int M, int N);
// targets with an id (not -1) -> *n_valid; other out-of-range ids raise the token bit
int count_targets(const int32_t* tgt, int M, int vocab_real, int* n_valid, int* err, cudaStream_t st);
// cross-entropy: logits [M, V] (act) -> in place dz = (softmax - onehot) M / n_valid
// (zero rows where the target is -1); loss_rows [M] (0 where masked)
int ce_fwd(int f32, void* logits, const int32_t* tgt, float* loss_rows, int M, int V,
           int vocab_real, const int* n_valid, int* err, cudaStream_t st);
int loss_mean(const float* loss_rows, int M, const int* n_valid, float* loss, int* err, cudaStream_t st);
// The cross-entropy from the LM head's EPI_CE_FWD outputs: per row the
// log-sum-exp (lse [M]) from the per-part maxima / sums [V/128][M], the loss row
// (LSE - z[target], 0 where masked), and, in place over the stored bf16
// exp(z - part max) [M, V], dz = (softmax - onehot(target)) * M / n_valid
// (zero rows where masked), the operand of the two backward GEMMs.
int ce_merge_dz(const float* part_max, const float* part_sum, const float* zt, const int32_t* tgt, void* e,
                float* lse, int M, int V, int vocab_real, const int* n_valid, float* loss_rows, cudaStream_t st);
// dwte[tok[m]] += dx[m] (deterministic fixed-point scatter at a resolution of
// 2^-32 |grad_scale|), dwpe (=/+=) sum_b dx
int embed_bwd(int f32, const int32_t* tok, const void* dx, float* dwte, float* dwpe,
              long long* acc, uint8_t* touched, int M, int T, int d, int V, int wpe_accumulate,
              float grad_scale, cudaStream_t st);
// AdamW over the flat buffer with the decay mask derived from the layout.
struct AdamArgs {
  float lr, beta1, beta2, eps, wd, bc1, bc2;
};
struct LayoutDims {
  long V, T, d, L;
};
// gnorm (device scalar, may be NULL): clip the gradient to global norm max_norm.
// Updates elements [base, base + n) of the flat buffers (base, n multiples of 4).
int adamw(float* p, const float* g, float* m, float* v, uint16_t* shadow, size_t n,
          const LayoutDims& ld, const AdamArgs& a, const float* gnorm, float max_norm, cudaStream_t st,
          size_t base = 0);
// ||g||_2 of n floats (n % 4 == 0) into *norm; part holds GRAD_NORM_PARTS floats.
constexpr int GRAD_NORM_PARTS = 592;
int grad_norm(const float* g, size_t n, float* part, float* norm, cudaStream_t st);
int init_params(float* p, size_t n, const LayoutDims& ld, uint64_t seed, cudaStream_t st);
int cast_shadow(const float* p, uint16_t* shadow, size_t n, cudaStream_t st);
int fill_zero(void* p, size_t bytes, cudaStream_t st);
int f32_to_act(int f32, const float* src, void* dst, long n, float scale, cudaStream_t st);

// ---- incremental decoding (key/value cache) -----------------------------
// One fused GEMV of the decode step: out[r, n] = epi(sum_k in'[r, k] W[n, k])
// for r < rows (<= 16), in' = the input row, LayerNorm'd first if ln.
enum DecodeEpiKind : int { DECODE_QKV = 0, DECODE_RESID = 1, DECODE_GELU = 2, DECODE_LOGITS = 3 };
struct DecodeGemv {
  const void* in;  // fp32 rows, or compute-dtype rows when in_t
  int in_t;
  const void* W;
  const void* bias;
  const void* ln_g;
  const void* ln_b;
  void* out;  // compute dtype for DECODE_GELU, else fp32
  long ldo;
  int rows, N, K;
  int ln, epi;
  void* kc;  // DECODE_QKV: this layer's K and V cache planes
  void* vc;
  const int32_t* pos;
  int d, H, hd, max_len;
};
size_t decode_gemv_smem(int f32, int rows, int K);
int decode_gemv(int f32, const DecodeGemv& g, cudaStream_t st);
int decode_embed(int f32, const int32_t* tok, const int32_t* pos, const void* wte, const void* wpe, float* x,
                 int rows, int d, int vocab_real, int limit, int* err, cudaStream_t st);
int decode_attention(int f32, const void* kc, const void* vc, const float* q, float* o, const int32_t* pos,
                     int rows, int H, int hd, int max_len, cudaStream_t st);
// part_v / part_i: GREEDY_SPLIT_MAX_ROWS x 16 scratch (may be NULL: one block per row)
constexpr int GREEDY_SPLIT_MAX_ROWS = 16;
int decode_greedy(const float* logits, long ld, int rows, int vocab_real, int32_t* next, int32_t* pos,
                  float* part_v, int* part_i, cudaStream_t st);
int prefill_kv(int f32, const void* qkv, void* kc, void* vc, const int32_t* plen, int rows, int T, int H, int hd,
               int max_len, int limit, int* err, cudaStream_t st);
int prefill_logits(int f32, const void* logits, const int32_t* plen, float* out, int rows, int T, int V, int limit,
                   cudaStream_t st);
