// C ABI of libgpt2.so: parameter layout, workspace carving, and the sequence
// of kernels that makes one GPT-2 training step (forward + loss, backward,
// AdamW).  Everything here runs on the host and only enqueues work.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace {

enum LayerTensor { LN1_G, LN1_B, W_QKV, B_QKV, W_O, B_O, LN2_G, LN2_B, W_FC, B_FC, W_MP, B_MP, N_LT };
const char* const kLayerNames[N_LT] = {"ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                                       "ln2_g", "ln2_b", "w_fc", "b_fc", "w_mp", "b_mp"};

struct Shape {
  long L, d, H, T, V, Vr, hd;
  int mode;  // 0 bf16, 1 fp32 (the configuration's mode 2 is bf16 with det set)
  bool det;  // bf16 with the attention backward's dQ summed in a fixed order
};

void lt_dims(long d, int t, long* rows, long* cols) {
  switch (t) {
    case W_QKV: *rows = 3 * d; *cols = d; return;
    case B_QKV: *rows = 3 * d; *cols = 1; return;
    case W_O: *rows = d; *cols = d; return;
    case W_FC: *rows = 4 * d; *cols = d; return;
    case B_FC: *rows = 4 * d; *cols = 1; return;
    case W_MP: *rows = d; *cols = 4 * d; return;
    default: *rows = d; *cols = 1; return;
  }
}
long lt_offset(long d, int t) {
  long off = 0;
  for (int i = 0; i < t; ++i) {
    long r, c;
    lt_dims(d, i, &r, &c);
    off += r * c;
  }
  return off;
}
long layer_size(long d) { return lt_offset(d, N_LT); }

struct Offsets {
  Shape s;
  size_t wte() const { return 0; }
  size_t wpe() const { return (size_t)(s.V * s.d); }
  size_t layer(int l, int t) const {
    return (size_t)((s.V + s.T) * s.d + l * layer_size(s.d) + lt_offset(s.d, t));
  }
  size_t lnf_g() const { return (size_t)((s.V + s.T) * s.d + s.L * layer_size(s.d)); }
  size_t lnf_b() const { return lnf_g() + s.d; }
  size_t total() const { return lnf_b() + s.d; }
};

bool shape_from_cfg(const gpt2_config* c, Shape* s) {
  if (!c) return false;
  if (c->n_layer < 1 || c->d_model < 1 || c->n_head < 1 || c->n_ctx < 1 || c->vocab_real < 1 ||
      c->vocab_padded < c->vocab_real || c->max_batch < 1 || c->mode < 0 || c->mode > 2)
    return false;
  if (c->d_model % c->n_head) return false;
  s->L = c->n_layer; s->d = c->d_model; s->H = c->n_head; s->T = c->n_ctx;
  s->V = c->vocab_padded; s->Vr = c->vocab_real; s->hd = c->d_model / c->n_head;
  s->mode = c->mode == 1 ? 1 : 0;
  s->det = c->mode == 2;
  return true;
}

int check_supported(const Shape& s, int max_batch) {
  if (s.d % 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (s.V % 128) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (s.hd != 16 && s.hd != 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (s.d > 2048) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (s.mode == 1 && s.T > 4096) return GPT2_ERR_UNSUPPORTED_SHAPE;
  // the fixed-order dQ sum is a mode of the tensor-core attention backward
  if (s.det && (s.hd != 64 || s.T > 4096)) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if ((long)max_batch * s.T > (1L << 30)) return GPT2_ERR_UNSUPPORTED_SHAPE;
  return GPT2_OK;
}

// Bump allocator over the workspace (base may be NULL to only measure).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <typename P>
  P* take(size_t bytes) {
    off = (off + 255) & ~(size_t)255;
    P* p = base ? reinterpret_cast<P*>(base + off) : nullptr;
    off += bytes;
    return p;
  }
};

struct LayerActs {
  // gp = GELU'(u) of the MLP pre-activation u (all the backward needs of u), g = GELU(u)
  void *x_in, *x_mid, *y1, *qkv, *o, *y2, *gp, *g;
  float *mean1, *rstd1, *mean2, *rstd2, *lse;
};

struct Work {
  int* err;
  float* loss;
  int32_t *tok, *tgt, *tok_stage, *tgt_stage;
  int32_t *gtok, *gtgt;  // inputs of the captured step
  std::vector<LayerActs> layers;
  void *x_final, *yf, *logits;
  float *meanf, *rstdf, *loss_rows;
  // fused cross-entropy (bf16): per-part maxima and sums [V/128][M], target
  // logits, row log-sum-exps
  float *ce_pm, *ce_ps, *ce_zt, *ce_lse;
  void *dres, *dy, *du, *dqkv, *dout;
  float *dq_acc, *dvec;
  float* dq_part;  // deterministic mode: per-key-block dQ tiles [T/128][M][d]
  float *norm_part, *gnorm;  // global gradient norm: block partials and the result
  int* n_valid;              // positions with a target in the last forward
  float* greedy_v;           // per-slice best (value, id) of the greedy choice
  int* greedy_i;
  // block partials of every bias / LayerNorm parameter gradient of one
  // backward, each in its own slot, all reduced by one launch at its end
  float* part_arena;
  size_t part_floats, part_used;
  std::vector<ReduceJob> jobs;
  void* split_ws;
  size_t split_bytes;
  int* split_cnt;  // per-tile split-order counters, zeroed at each backward
  long long* emb_acc;
  uint8_t* touched;
};

// The LM head's input-gradient GEMM (M x d, K = V) has only M/256 * d/256
// output tiles (192 at the 124M shape) for 74 SM pairs, 2.6 waves; three
// K splits make 7.8 waves of a third of the work each.
constexpr int LM_DGRAD_SPLITS = 3;
// Counters of the in-kernel split-K ordering: one per (tile, CTA, epilogue
// warp); split-K is chosen only with fewer tiles than SM pairs or SMs.
constexpr int SPLIT_COUNTERS = 4096;

size_t split_ws_need(const Shape& s, long M) {
  if (s.mode != 0) return 0;
  size_t need = 0;
  const long d = s.d;
  const long shapes[5][2] = {{3 * d, d}, {d, d}, {4 * d, d}, {d, 4 * d}, {s.V, d}};
  for (auto& sh : shapes) {
    size_t b = gemm_tc_split_bytes((int)sh[0], (int)sh[1], (int)M);
    if (b > need) need = b;
  }
  // the LM head's input gradient, split along the vocabulary
  const size_t lm = (size_t)LM_DGRAD_SPLITS * M * d * sizeof(float);
  return need > lm ? need : lm;
}

size_t carve(const Shape& s, int batch, uint8_t* base, Work* w) {
  Carver c{base};
  const long M = (long)batch * s.T, d = s.d;
  const size_t act = s.mode ? 4 : 2;
  w->err = c.take<int>(sizeof(int));
  w->loss = c.take<float>(sizeof(float));
  w->tok = c.take<int32_t>(M * 4);
  w->tgt = c.take<int32_t>(M * 4);
  // the captured step's inputs (copied in by gpt2_graph_step)
  w->gtok = c.take<int32_t>(M * 4);
  w->gtgt = c.take<int32_t>(M * 4);
  w->tok_stage = c.take<int32_t>(M * 4);
  w->tgt_stage = c.take<int32_t>(M * 4);
  w->layers.assign(s.L, LayerActs{});
  void* x_prev = c.take<void>(M * d * act);  // x_0: the embedding output
  for (long l = 0; l < s.L; ++l) {
    LayerActs& a = w->layers[l];
    a.x_in = x_prev;
    a.y1 = c.take<void>(M * d * act);
    a.mean1 = c.take<float>(M * 4);
    a.rstd1 = c.take<float>(M * 4);
    a.qkv = c.take<void>(M * 3 * d * act);
    a.o = c.take<void>(M * d * act);
    a.lse = c.take<float>(M * s.H * 4);
    a.x_mid = c.take<void>(M * d * act);
    a.y2 = c.take<void>(M * d * act);
    a.mean2 = c.take<float>(M * 4);
    a.rstd2 = c.take<float>(M * 4);
    a.gp = c.take<void>(M * 4 * d * act);
    a.g = c.take<void>(M * 4 * d * act);
    x_prev = c.take<void>(M * d * act);
  }
  w->x_final = x_prev;
  w->yf = c.take<void>(M * d * act);
  w->meanf = c.take<float>(M * 4);
  w->rstdf = c.take<float>(M * 4);
  w->logits = c.take<void>(M * s.V * act);
  w->loss_rows = c.take<float>(M * 4);
  const long parts = s.V / 128;
  w->ce_pm = c.take<float>((size_t)parts * M * 4);
  w->ce_ps = c.take<float>((size_t)parts * M * 4);
  w->ce_zt = c.take<float>(M * 4);
  w->ce_lse = c.take<float>(M * 4);
  w->dres = c.take<void>(M * d * act);
  w->dy = c.take<void>(M * d * act);
  w->du = c.take<void>(M * 4 * d * act);
  w->dqkv = c.take<void>(M * 3 * d * act);
  w->dout = c.take<void>(M * d * act);
  w->dq_acc = c.take<float>(M * d * 4);
  w->dq_part = s.det ? c.take<float>((size_t)((s.T + 127) / 128) * M * d * 4) : nullptr;
  w->dvec = c.take<float>(M * s.H * 4);
  // per layer: two LayerNorms (gamma/beta partials + the column sums of their
  // output, the b_o / b_mp gradients) and the b_fc, b_qkv column sums; plus
  // the final LayerNorm
  const size_t ln_rows = layernorm_bwd_part_rows((int)M);
  // (the b_fc sums come from the GELU' GEMM's epilogue, one row per 32 tokens,
  // on the tensor-core path)
  const size_t fc_part = std::max(colsum_part_floats((int)M, (int)(4 * d)), (size_t)((M + 31) / 32) * 4 * d);
  w->part_floats = (size_t)s.L * (2 * ln_rows * 3 * d + fc_part + colsum_part_floats((int)M, (int)(3 * d))) +
                   ln_rows * 3 * d;
  w->part_arena = c.take<float>(w->part_floats * 4);
  w->norm_part = c.take<float>((size_t)GRAD_NORM_PARTS * 4);
  w->gnorm = c.take<float>(4);
  w->n_valid = c.take<int>(4);
  w->greedy_v = c.take<float>((size_t)GREEDY_SPLIT_MAX_ROWS * 16 * 4);
  w->greedy_i = c.take<int>((size_t)GREEDY_SPLIT_MAX_ROWS * 16 * 4);
  w->part_used = 0;
  w->split_bytes = split_ws_need(s, M);
  w->split_ws = c.take<void>(w->split_bytes);
  w->split_cnt = c.take<int>(SPLIT_COUNTERS * sizeof(int));
  w->emb_acc = c.take<long long>((size_t)s.V * d * 8);
  w->touched = c.take<uint8_t>((size_t)s.V);
  return (c.off + 255) & ~(size_t)255;
}

}  // namespace

static std::atomic<unsigned long long> g_launches{0};
void gpt2_count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

struct gpt2_ctx {
  gpt2_config cfg;
  Shape s;
  Offsets off;
  gpt2_buffers buf;
  Work w;
  int have_fwd = 0;
  int fwd_batch = 0;
  // the captured micro-step (gpt2_graph_capture)
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t graph_exec = nullptr;
  int graph_batch = 0;
  int graph_plain = 0;  // captured with grad_scale 1, accumulate 0
  float* graph_loss = nullptr;  // where the graph writes the loss
  unsigned long long graph_launches = 0;  // kernels in one launch of the graph
  ~gpt2_ctx() {
    if (graph_exec) cudaGraphExecDestroy(graph_exec);
    if (graph) cudaGraphDestroy(graph);
  }
};

namespace {

cudaStream_t S(void* st) { return reinterpret_cast<cudaStream_t>(st); }

// Parameter pointers in the compute dtype: bf16 shadow (mode 0) or fp32 master.
const void* Wp(const gpt2_ctx* c, size_t off) {
  return c->s.mode ? (const void*)(c->buf.master + off) : (const void*)(c->buf.shadow + off);
}

int run_gemm(gpt2_ctx* c, const GemmArgs& g, cudaStream_t st) {
  if (c->s.mode) return gemm_simt_f32(g, st);
  GemmArgs h = g;
  // weight gradients split along K are reduced inside the kernel, in order
  h.epi.split_cnt = c->w.split_cnt;
  h.epi.split_cnt_len = SPLIT_COUNTERS;
  return gemm_tc_bf16(h, c->w.split_ws, c->w.split_bytes, 0, 0, c->w.err, st);
}

GemmArgs make_gemm(int M, int N, int K, const void* A, int a_mn, long lda, const void* B, int b_mn, long ldb,
                   int kind, void* out, long ldo) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.M = M; g.N = N; g.K = K;
  g.A = A; g.a_mn = a_mn; g.lda = lda;
  g.B = B; g.b_mn = b_mn; g.ldb = ldb;
  g.epi.kind = kind;
  g.epi.out = out;
  g.epi.ldo = ldo;
  g.epi.alpha = 1.f;
  g.epi.beta = 0.f;
  return g;
}

#define TRY(x)              \
  do {                      \
    int rc_ = (x);          \
    if (rc_) return rc_;    \
  } while (0)

// A slot of the partials arena (sized in carve for every slot of a backward).
float* part_slot(gpt2_ctx* c, size_t floats) {
  float* p = c->w.part_arena + c->w.part_used;
  c->w.part_used += floats;
  return p;
}
// param grads of one (gamma, beta) pair / bias: block partials now, the
// reduction queued for the batched launch that ends the backward
void ln_param_grads(gpt2_ctx* c, const float* part, int nblk, size_t goff) {
  c->w.jobs.push_back(ReduceJob{part, c->buf.grad + goff, nblk, (int)(2 * c->s.d)});
}
// LayerNorm backward writing the new residual-stream gradient into w.dres,
// its (gamma, beta) gradient at goff and, when res_goff is not ~0, the column
// sums of that new gradient (a bias gradient) at res_goff
int ln_backward(gpt2_ctx* c, const void* x, const float* mean, const float* rstd, size_t g_off, int init,
                size_t goff, size_t res_goff, int M, cudaStream_t st) {
  const int d = (int)c->s.d;
  const size_t rows = layernorm_bwd_part_rows(M);
  float* part = part_slot(c, rows * 2 * d);
  float* pres = res_goff != ~(size_t)0 ? part_slot(c, rows * d) : nullptr;
  int nblk = 0;
  TRY(layernorm_bwd(c->s.mode, c->w.dy, x, mean, rstd, Wp(c, g_off), c->w.dres, init, part, pres, &nblk, M, d,
                    st));
  ln_param_grads(c, part, nblk, goff);
  if (pres) c->w.jobs.push_back(ReduceJob{pres, c->buf.grad + res_goff, nblk, d});
  return GPT2_OK;
}
int bias_grad(gpt2_ctx* c, const void* x, int M, int N, size_t goff, cudaStream_t st) {
  int nblk = 0;
  float* part = part_slot(c, colsum_part_floats(M, N));
  TRY(colsum_partial(c->s.mode, x, M, N, part, &nblk, st));
  c->w.jobs.push_back(ReduceJob{part, c->buf.grad + goff, nblk, N});
  return GPT2_OK;
}

}  // namespace

extern "C" {

size_t gpt2_param_count(const gpt2_config* cfg) {
  Shape s;
  if (!shape_from_cfg(cfg, &s)) return 0;
  Offsets o{s};
  return o.total();
}

size_t gpt2_workspace_bytes(const gpt2_config* cfg, int batch) {
  Shape s;
  if (!shape_from_cfg(cfg, &s) || batch < 1) return 0;
  Work w;
  return carve(s, batch, nullptr, &w);
}

int gpt2_tensor_info(const gpt2_config* cfg, int index, const char** name, size_t* offset, size_t* rows,
                     size_t* cols) {
  static char namebuf[64];
  Shape s;
  if (!shape_from_cfg(cfg, &s) || index < 0) return GPT2_ERR_INVALID_ARG;
  Offsets o{s};
  long r = 0, cc = 1;
  size_t off = 0;
  const int nl = (int)s.L * N_LT;
  if (index == 0) {
    snprintf(namebuf, sizeof(namebuf), "wte"); off = o.wte(); r = s.V; cc = s.d;
  } else if (index == 1) {
    snprintf(namebuf, sizeof(namebuf), "wpe"); off = o.wpe(); r = s.T; cc = s.d;
  } else if (index < 2 + nl) {
    int l = (index - 2) / N_LT, t = (index - 2) % N_LT;
    snprintf(namebuf, sizeof(namebuf), "h%d.%s", l, kLayerNames[t]);
    off = o.layer(l, t);
    lt_dims(s.d, t, &r, &cc);
  } else if (index == 2 + nl) {
    snprintf(namebuf, sizeof(namebuf), "lnf_g"); off = o.lnf_g(); r = s.d;
  } else if (index == 3 + nl) {
    snprintf(namebuf, sizeof(namebuf), "lnf_b"); off = o.lnf_b(); r = s.d;
  } else {
    return GPT2_ERR_INVALID_ARG;
  }
  if (name) *name = namebuf;
  if (offset) *offset = off;
  if (rows) *rows = (size_t)r;
  if (cols) *cols = (size_t)cc;
  return GPT2_OK;
}

int gpt2_create(const gpt2_config* cfg, const gpt2_buffers* bufs, gpt2_ctx** out) {
  if (!cfg || !bufs || !out) return GPT2_ERR_INVALID_ARG;
  *out = nullptr;
  Shape s;
  if (!shape_from_cfg(cfg, &s)) return GPT2_ERR_INVALID_ARG;
  TRY(check_supported(s, cfg->max_batch));
  if (s.mode == 0 && ((long)cfg->max_batch * s.T) % 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (!bufs->master || !bufs->grad || !bufs->m || !bufs->v || !bufs->workspace) return GPT2_ERR_INVALID_ARG;
  if (s.mode == 0 && !bufs->shadow) return GPT2_ERR_INVALID_ARG;
  const uintptr_t align = (uintptr_t)bufs->master | (uintptr_t)bufs->grad | (uintptr_t)bufs->m |
                          (uintptr_t)bufs->v | (uintptr_t)bufs->workspace | (uintptr_t)bufs->shadow;
  if (align & 15) return GPT2_ERR_INVALID_ARG;
  gpt2_ctx* c = new gpt2_ctx();
  c->cfg = *cfg;
  c->s = s;
  c->off = Offsets{s};
  c->buf = *bufs;
  const size_t need = carve(s, cfg->max_batch, (uint8_t*)bufs->workspace, &c->w);
  if (bufs->workspace_bytes < need) {
    delete c;
    return GPT2_ERR_WORKSPACE;
  }
  if (cudaMemset(c->w.err, 0, sizeof(int)) != cudaSuccess ||
      cudaMemset(c->w.emb_acc, 0, (size_t)s.V * s.d * 8) != cudaSuccess ||
      cudaMemset(c->w.touched, 0, (size_t)s.V) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    delete c;
    return GPT2_ERR_CUDA;
  }
  *out = c;
  return GPT2_OK;
}

int gpt2_destroy(gpt2_ctx* ctx) {
  delete ctx;
  return GPT2_OK;
}

int gpt2_refresh_shadow(gpt2_ctx* c, void* stream) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  if (!c->buf.shadow) return GPT2_OK;
  return cast_shadow(c->buf.master, c->buf.shadow, c->off.total(), S(stream));
}

int gpt2_init_params(gpt2_ctx* c, uint64_t seed, void* stream) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  const size_t n = c->off.total();
  LayoutDims ld{c->s.V, c->s.T, c->s.d, c->s.L};
  TRY(init_params(c->buf.master, n, ld, seed, S(stream)));
  TRY(fill_zero(c->buf.grad, n * 4, S(stream)));
  TRY(fill_zero(c->buf.m, n * 4, S(stream)));
  TRY(fill_zero(c->buf.v, n * 4, S(stream)));
  return gpt2_refresh_shadow(c, stream);
}

int gpt2_zero_grad(gpt2_ctx* c, void* stream) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  return fill_zero(c->buf.grad, c->off.total() * 4, S(stream));
}

namespace {

// The forward up to the LM head; every layer's activations stay in the
// workspace.  Plain: the logits [batch * T, V] in w.logits.  ce_fused (bf16):
// the LM-head GEMM computes the cross-entropy's per-part maxima and sums of
// exp(z - max) in its epilogue and stores those exponentials (bf16) in
// w.logits instead of z, plus the target logits (w.tgt must hold the targets).
int forward_logits(gpt2_ctx* c, const int32_t* tokens, int batch, cudaStream_t st, bool ce_fused = false) {
  const Shape& s = c->s;
  const int M = batch * (int)s.T, d = (int)s.d, V = (int)s.V;
  Work& w = c->w;
  const Offsets& o = c->off;
  const int f32 = s.mode;
  CUDA_TRY(cudaMemcpyAsync(w.tok, tokens, (size_t)M * 4, cudaMemcpyDeviceToDevice, st));
  c->have_fwd = 0;

  TRY(embed_fwd(f32, w.tok, Wp(c, o.wte()), Wp(c, o.wpe()), w.layers[0].x_in, M, (int)s.T, d, (int)s.Vr, w.err,
                st));
  for (int l = 0; l < (int)s.L; ++l) {
    LayerActs& a = w.layers[l];
    TRY(layernorm_fwd(f32, a.x_in, Wp(c, o.layer(l, LN1_G)), Wp(c, o.layer(l, LN1_B)), a.y1, a.mean1, a.rstd1, M,
                      d, st));
    GemmArgs g = make_gemm(M, 3 * d, d, a.y1, 0, d, Wp(c, o.layer(l, W_QKV)), 0, d, EPI_BIAS, a.qkv, 3 * d);
    g.epi.bias = Wp(c, o.layer(l, B_QKV));
    TRY(run_gemm(c, g, st));
    if (f32)
      TRY(attn_fwd_f32((const float*)a.qkv, (float*)a.o, a.lse, batch, (int)s.T, (int)s.H, (int)s.hd, st));
    else
      TRY(attn_fwd_bf16(a.qkv, a.o, a.lse, batch, (int)s.T, (int)s.H, (int)s.hd, st));
    g = make_gemm(M, d, d, a.o, 0, d, Wp(c, o.layer(l, W_O)), 0, d, EPI_BIAS_RESID, a.x_mid, d);
    g.epi.bias = Wp(c, o.layer(l, B_O));
    g.epi.resid = a.x_in;
    TRY(run_gemm(c, g, st));
    TRY(layernorm_fwd(f32, a.x_mid, Wp(c, o.layer(l, LN2_G)), Wp(c, o.layer(l, LN2_B)), a.y2, a.mean2, a.rstd2,
                      M, d, st));
    g = make_gemm(M, 4 * d, d, a.y2, 0, d, Wp(c, o.layer(l, W_FC)), 0, d, EPI_BIAS_GELU, a.gp, 4 * d);
    g.epi.bias = Wp(c, o.layer(l, B_FC));
    g.epi.out2 = a.g;
    TRY(run_gemm(c, g, st));
    void* x_out = (l + 1 < (int)s.L) ? w.layers[l + 1].x_in : w.x_final;
    g = make_gemm(M, d, 4 * d, a.g, 0, 4 * d, Wp(c, o.layer(l, W_MP)), 0, 4 * d, EPI_BIAS_RESID, x_out, d);
    g.epi.bias = Wp(c, o.layer(l, B_MP));
    g.epi.resid = a.x_mid;
    TRY(run_gemm(c, g, st));
  }
  TRY(layernorm_fwd(f32, w.x_final, Wp(c, o.lnf_g()), Wp(c, o.lnf_b()), w.yf, w.meanf, w.rstdf, M, d, st));
  GemmArgs g = make_gemm(M, V, d, w.yf, 0, d, Wp(c, o.wte()), 0, d, ce_fused ? EPI_CE_FWD : EPI_STORE, w.logits, V);
  if (ce_fused) {
    g.epi.ce_max = w.ce_pm;
    g.epi.ce_sum = w.ce_ps;
    g.epi.ce_zt = w.ce_zt;
    g.epi.ce_tgt = w.tgt;
  }
  TRY(run_gemm(c, g, st));
  return GPT2_OK;
}

}  // namespace

int gpt2_forward_loss(gpt2_ctx* c, const int32_t* tokens, const int32_t* targets, int batch, float* loss_dev,
                      void* stream) {
  if (!c || !tokens || !targets) return GPT2_ERR_INVALID_ARG;
  if (batch < 1 || batch > c->cfg.max_batch) return GPT2_ERR_INVALID_ARG;
  const Shape& s = c->s;
  const int M = batch * (int)s.T, V = (int)s.V;
  if (s.mode == 0 && M % 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = S(stream);
  Work& w = c->w;
  const int f32 = s.mode;
  CUDA_TRY(cudaMemcpyAsync(w.tgt, targets, (size_t)M * 4, cudaMemcpyDeviceToDevice, st));
  TRY(forward_logits(c, tokens, batch, st, !f32));
  TRY(count_targets(w.tgt, M, (int)s.Vr, w.n_valid, w.err, st));
  if (f32)
    TRY(ce_fwd(f32, w.logits, w.tgt, w.loss_rows, M, V, (int)s.Vr, w.n_valid, w.err, st));
  else
    TRY(ce_merge_dz(w.ce_pm, w.ce_ps, w.ce_zt, w.tgt, w.logits, w.ce_lse, M, V, (int)s.Vr, w.n_valid, w.loss_rows,
                    st));
  TRY(loss_mean(w.loss_rows, M, w.n_valid, loss_dev ? loss_dev : w.loss, w.err, st));
  c->have_fwd = 1;
  c->fwd_batch = batch;
  return GPT2_OK;
}

}  // extern "C"

namespace {

// The backward.  With events (L + 2 of them) the gradients are finished in
// buckets and each bucket's event is recorded on the stream as soon as its
// gradients are final: events[l] for layer l's block, events[L] for the final
// LayerNorm, events[L + 1] for the token and position embeddings (the tied
// wte gradient takes the embedding scatter last).  The block partials of the
// bias and LayerNorm gradients are then reduced per bucket instead of in one
// launch at the end.
int backward_impl(gpt2_ctx* c, float grad_scale, int accumulate, void* const* events, void* stream) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  if (!c->have_fwd) return GPT2_ERR_BAD_STATE;
  const Shape& s = c->s;
  const int batch = c->fwd_batch;
  const int M = batch * (int)s.T, d = (int)s.d, V = (int)s.V;
  cudaStream_t st = S(stream);
  Work& w = c->w;
  const Offsets& o = c->off;
  const int f32 = s.mode;
  const float beta = accumulate ? 1.f : 0.f;
  const float sc = grad_scale / (float)M;
  float* G = c->buf.grad;
  // D = rowsum(dO * O) fused into the attention projection's input-gradient
  // GEMM (tensor-core path, head_dim 64); dq_acc then starts zeroed here and
  // every attention backward leaves it zeroed
  const int fuse_d = (!f32 && s.hd == 64) ? 1 : 0;
  if (fuse_d) TRY(fill_zero(w.dq_acc, (size_t)M * d * sizeof(float), st));
  // the split-order counters start at zero (each reduction also leaves them
  // so; this also clears what an aborted launch may have left)
  if (!f32) TRY(fill_zero(w.split_cnt, SPLIT_COUNTERS * sizeof(int), st));

  // LM head (tied): dX_f = s * dz wte ; dwte (=/+=) s * dz^T X_f, with dz =
  // (softmax - onehot) M / n_valid left in w.logits by the forward
  GemmArgs g = make_gemm(M, d, V, w.logits, 0, V, Wp(c, o.wte()), 1, d, EPI_STORE, w.dy, d);
  g.epi.alpha = sc;
  if (f32)
    TRY(run_gemm(c, g, st));
  else
    TRY(gemm_tc_bf16(g, w.split_ws, w.split_bytes, 0, LM_DGRAD_SPLITS, w.err, st));
  g = make_gemm(V, d, M, w.logits, 1, V, w.yf, 1, d, EPI_F32, G + o.wte(), d);
  g.epi.alpha = sc;
  g.epi.beta = beta;
  TRY(run_gemm(c, g, st));
  w.part_used = 0;
  w.jobs.clear();
  // the new residual gradient's column sums are the last MLP projection's b_mp gradient
  TRY(ln_backward(c, w.x_final, w.meanf, w.rstdf, o.lnf_g(), 1, o.lnf_g(), o.layer(s.L - 1, B_MP), M, st));
  // bucketed: reduce every pending job except the last (it belongs to the next
  // bucket, the block below), then mark the bucket
  size_t flushed = 0;
  auto flush_bucket = [&](size_t keep, void* ev) -> int {
    const size_t upto = w.jobs.size() - keep;
    if (upto > flushed) TRY(reduce_rows_batch(w.jobs.data() + flushed, (int)(upto - flushed), beta, st));
    flushed = upto;
    if (ev) CUDA_TRY(cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), st));
    return GPT2_OK;
  };
  if (events) TRY(flush_bucket(1, events[s.L]));

  for (int l = (int)s.L - 1; l >= 0; --l) {
    LayerActs& a = w.layers[l];
    // MLP projection: x_out = x_mid + g W_mp^T + b_mp
    g = make_gemm(M, 4 * d, d, w.dres, 0, d, Wp(c, o.layer(l, W_MP)), 1, 4 * d, EPI_DGELU, w.du, 4 * d);
    g.epi.aux = a.gp;
    // b_fc gradient partials (column sums of du per 32 rows) from the same epilogue
    float* fc_part = f32 ? nullptr : part_slot(c, (size_t)((M + 31) / 32) * 4 * d);
    g.epi.colsum = fc_part;
    TRY(run_gemm(c, g, st));
    g = make_gemm(d, 4 * d, M, w.dres, 1, d, a.g, 1, 4 * d, EPI_F32, G + o.layer(l, W_MP), 4 * d);
    g.epi.beta = beta;
    TRY(run_gemm(c, g, st));
    // MLP fc: u = y2 W_fc^T + b_fc
    g = make_gemm(M, d, 4 * d, w.du, 0, 4 * d, Wp(c, o.layer(l, W_FC)), 1, d, EPI_STORE, w.dy, d);
    TRY(run_gemm(c, g, st));
    g = make_gemm(4 * d, d, M, w.du, 1, 4 * d, a.y2, 1, d, EPI_F32, G + o.layer(l, W_FC), d);
    g.epi.beta = beta;
    TRY(run_gemm(c, g, st));
    if (fc_part)
      w.jobs.push_back(ReduceJob{fc_part, G + o.layer(l, B_FC), (M + 31) / 32, 4 * d});
    else
      TRY(bias_grad(c, w.du, M, 4 * d, o.layer(l, B_FC), st));
    // column sums of the new residual gradient: the attention projection's b_o gradient
    TRY(ln_backward(c, a.x_mid, a.mean2, a.rstd2, o.layer(l, LN2_G), 0, o.layer(l, LN2_G), o.layer(l, B_O), M, st));
    // attention projection: x_mid = x_in + o W_o^T + b_o
    // (bf16, head_dim 64: the epilogue also writes D = rowsum(dO * O) per head,
    // the attention backward's first input)
    g = make_gemm(M, d, d, w.dres, 0, d, Wp(c, o.layer(l, W_O)), 1, d, fuse_d ? EPI_ROWDOT : EPI_STORE, w.dout, d);
    if (fuse_d) {
      g.epi.aux = a.o;
      g.epi.out2 = w.dvec;
      g.epi.seq = (int)s.T;
    }
    TRY(run_gemm(c, g, st));
    g = make_gemm(d, d, M, w.dres, 1, d, a.o, 1, d, EPI_F32, G + o.layer(l, W_O), d);
    g.epi.beta = beta;
    TRY(run_gemm(c, g, st));
    // attention
    if (f32)
      TRY(attn_bwd_f32((const float*)a.qkv, (const float*)a.o, a.lse, (const float*)w.dout, (float*)w.dqkv, w.dvec,
                       batch, (int)s.T, (int)s.H, (int)s.hd, st));
    else
      TRY(attn_bwd_bf16(a.qkv, a.o, a.lse, w.dout, w.dqkv, w.dq_acc, w.dvec, batch, (int)s.T, (int)s.H, (int)s.hd,
                        st, fuse_d, w.dq_part));
    // QKV: qkv = y1 W_qkv^T + b_qkv
    g = make_gemm(M, d, 3 * d, w.dqkv, 0, 3 * d, Wp(c, o.layer(l, W_QKV)), 1, d, EPI_STORE, w.dy, d);
    TRY(run_gemm(c, g, st));
    g = make_gemm(3 * d, d, M, w.dqkv, 1, 3 * d, a.y1, 1, d, EPI_F32, G + o.layer(l, W_QKV), d);
    g.epi.beta = beta;
    TRY(run_gemm(c, g, st));
    TRY(bias_grad(c, w.dqkv, M, 3 * d, o.layer(l, B_QKV), st));
    // column sums of the new residual gradient: the previous layer's b_mp gradient
    TRY(ln_backward(c, a.x_in, a.mean1, a.rstd1, o.layer(l, LN1_G), 0, o.layer(l, LN1_G),
                    l > 0 ? o.layer(l - 1, B_MP) : ~(size_t)0, M, st));
    // layer l's gradients are final once its partials are reduced (the last
    // job is layer l-1's b_mp)
    if (events) TRY(flush_bucket(l > 0 ? 1 : 0, events[l]));
  }
  // every (remaining) bias and LayerNorm parameter gradient, in one launch
  if (w.jobs.size() > flushed)
    TRY(reduce_rows_batch(w.jobs.data() + flushed, (int)(w.jobs.size() - flushed), beta, st));
  // x_0 = wte[tok] + wpe[t]
  TRY(embed_bwd(f32, w.tok, w.dres, G + o.wte(), G + o.wpe(), w.emb_acc, w.touched, M, (int)s.T, d, V, accumulate,
                grad_scale, st));
  if (events) CUDA_TRY(cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[s.L + 1]), st));
  return GPT2_OK;
}

}  // namespace

extern "C" {

int gpt2_backward(gpt2_ctx* c, float grad_scale, int accumulate, void* stream) {
  return backward_impl(c, grad_scale, accumulate, nullptr, stream);
}

int gpt2_backward_bucketed(gpt2_ctx* c, float grad_scale, int accumulate, void* const* events, int n_events,
                           void* stream) {
  if (!c || !events) return GPT2_ERR_INVALID_ARG;
  if (n_events != (int)c->s.L + 2) return GPT2_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return GPT2_ERR_INVALID_ARG;
  return backward_impl(c, grad_scale, accumulate, events, stream);
}

int gpt2_adamw_step(gpt2_ctx* c, float lr, float beta1, float beta2, float eps, float weight_decay, int step,
                    void* stream) {
  if (!c || step < 1) return GPT2_ERR_INVALID_ARG;
  AdamArgs a;
  a.lr = lr; a.beta1 = beta1; a.beta2 = beta2; a.eps = eps; a.wd = weight_decay;
  a.bc1 = (float)(1.0 - pow((double)beta1, (double)step));
  a.bc2 = (float)(1.0 - pow((double)beta2, (double)step));
  LayoutDims ld{c->s.V, c->s.T, c->s.d, c->s.L};
  return adamw(c->buf.master, c->buf.grad, c->buf.m, c->buf.v, c->s.mode ? nullptr : c->buf.shadow,
               c->off.total(), ld, a, nullptr, 0.f, S(stream));
}

int gpt2_adamw_step_range(gpt2_ctx* c, float lr, float beta1, float beta2, float eps, float weight_decay,
                          int step, size_t offset, size_t count, void* stream) {
  if (!c || step < 1 || offset % 4 || count % 4 || offset > c->off.total() || count > c->off.total() - offset)
    return GPT2_ERR_INVALID_ARG;
  AdamArgs a;
  a.lr = lr; a.beta1 = beta1; a.beta2 = beta2; a.eps = eps; a.wd = weight_decay;
  a.bc1 = (float)(1.0 - pow((double)beta1, (double)step));
  a.bc2 = (float)(1.0 - pow((double)beta2, (double)step));
  LayoutDims ld{c->s.V, c->s.T, c->s.d, c->s.L};
  return adamw(c->buf.master, c->buf.grad, c->buf.m, c->buf.v, c->s.mode ? nullptr : c->buf.shadow, count, ld, a,
               nullptr, 0.f, S(stream), offset);
}

int gpt2_grad_norm(gpt2_ctx* c, float* norm_dev, void* stream) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  if (norm_dev && ((uintptr_t)norm_dev & 3)) return GPT2_ERR_INVALID_ARG;
  return grad_norm(c->buf.grad, c->off.total(), c->w.norm_part, norm_dev ? norm_dev : c->w.gnorm, S(stream));
}

int gpt2_adamw_step_clip(gpt2_ctx* c, float lr, float beta1, float beta2, float eps, float weight_decay, int step,
                         float max_norm, void* stream) {
  if (!c || step < 1 || !(max_norm >= 0.f)) return GPT2_ERR_INVALID_ARG;
  if (max_norm == 0.f) return gpt2_adamw_step(c, lr, beta1, beta2, eps, weight_decay, step, stream);
  int rc = grad_norm(c->buf.grad, c->off.total(), c->w.norm_part, c->w.gnorm, S(stream));
  if (rc) return rc;
  AdamArgs a;
  a.lr = lr; a.beta1 = beta1; a.beta2 = beta2; a.eps = eps; a.wd = weight_decay;
  a.bc1 = (float)(1.0 - pow((double)beta1, (double)step));
  a.bc2 = (float)(1.0 - pow((double)beta2, (double)step));
  LayoutDims ld{c->s.V, c->s.T, c->s.d, c->s.L};
  return adamw(c->buf.master, c->buf.grad, c->buf.m, c->buf.v, c->s.mode ? nullptr : c->buf.shadow,
               c->off.total(), ld, a, c->w.gnorm, max_norm, S(stream));
}

int gpt2_get_status(gpt2_ctx* c, void* stream) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return GPT2_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, c->w.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  if (h && cudaMemset(c->w.err, 0, sizeof(int)) != cudaSuccess) return GPT2_ERR_CUDA;
  if (h & DEV_ERR_TIMEOUT) return GPT2_ERR_TIMEOUT;
  if (h & DEV_ERR_NONFINITE) return GPT2_ERR_NONFINITE;
  if (h & DEV_ERR_TOKEN) return GPT2_ERR_TOKEN_RANGE;
  if (h & DEV_ERR_POSITION) return GPT2_ERR_POSITION_RANGE;
  return GPT2_OK;
}

// ------------------------------------------------ incremental decoding ----

namespace {

// The cache: K and V planes [batch][H][max_len][hd] (compute dtype) of every
// layer, layer-major (K of layer l, then V of layer l), then the decode
// step's fp32 rows x (residual stream), q, o [batch, d] and g [batch, 4d].
struct DecodeLayout {
  uint8_t* base = nullptr;
  size_t plane_bytes = 0;
  float *x = nullptr, *q = nullptr, *o = nullptr, *g = nullptr;
  size_t total = 0;
  void* k(int l) const { return base + (size_t)(2 * l) * plane_bytes; }
  void* v(int l) const { return base + (size_t)(2 * l + 1) * plane_bytes; }
};

constexpr int DECODE_MAX_BATCH = 16;

bool decode_layout(const Shape& s, int batch, int max_len, void* cache, DecodeLayout* dl) {
  if (batch < 1 || batch > DECODE_MAX_BATCH || max_len < 1 || max_len > s.T) return false;
  const size_t es = s.mode ? 4 : 2;
  dl->base = reinterpret_cast<uint8_t*>(cache);
  dl->plane_bytes = ((size_t)batch * s.H * max_len * s.hd * es + 255) & ~(size_t)255;
  size_t off = (size_t)(2 * s.L) * dl->plane_bytes;
  auto take = [&](size_t floats) {
    float* p = cache ? reinterpret_cast<float*>(dl->base + off) : nullptr;
    off += (floats * 4 + 255) & ~(size_t)255;
    return p;
  };
  dl->x = take((size_t)batch * s.d);
  dl->q = take((size_t)batch * s.d);
  dl->o = take((size_t)batch * s.d);
  dl->g = take((size_t)batch * 4 * s.d);
  dl->total = off;
  return true;
}

int decode_check(gpt2_ctx* c, void* cache, size_t cache_bytes, int batch, int max_len, DecodeLayout* dl) {
  if (!c || !cache || ((uintptr_t)cache & 255)) return GPT2_ERR_INVALID_ARG;
  if (!decode_layout(c->s, batch, max_len, cache, dl)) return GPT2_ERR_INVALID_ARG;
  if (dl->total > cache_bytes) return GPT2_ERR_INVALID_ARG;  // sized for another (batch, max_len)
  if (decode_gemv_smem(c->s.mode, batch, (int)(4 * c->s.d)) > 227 * 1024) return GPT2_ERR_UNSUPPORTED_SHAPE;
  return GPT2_OK;
}

}  // namespace

size_t gpt2_kv_cache_bytes(const gpt2_config* cfg, int batch, int max_len) {
  Shape s;
  DecodeLayout dl;
  if (!shape_from_cfg(cfg, &s) || !decode_layout(s, batch, max_len, nullptr, &dl)) return 0;
  return dl.total;
}

int gpt2_decode_step(gpt2_ctx* c, void* cache, size_t cache_bytes, int batch, int max_len, const int32_t* tokens,
                     const int32_t* pos, float* logits, void* stream) {
  DecodeLayout dl;
  TRY(decode_check(c, cache, cache_bytes, batch, max_len, &dl));
  if (!tokens || !pos || !logits) return GPT2_ERR_INVALID_ARG;
  const Shape& s = c->s;
  const Offsets& o = c->off;
  const int f32 = s.mode, d = (int)s.d;
  cudaStream_t st = S(stream);
  TRY(decode_embed(f32, tokens, pos, Wp(c, o.wte()), Wp(c, o.wpe()), dl.x, batch, d, (int)s.Vr, max_len, c->w.err,
                   st));
  DecodeGemv g;
  memset(&g, 0, sizeof(g));
  g.rows = batch;
  g.pos = pos;
  g.d = d; g.H = (int)s.H; g.hd = (int)s.hd; g.max_len = max_len;
  for (int l = 0; l < (int)s.L; ++l) {
    // LN1 -> QKV (+ bias): q to dl.q, k and v into the cache at pos
    g.in = dl.x; g.in_t = 0; g.W = Wp(c, o.layer(l, W_QKV)); g.bias = Wp(c, o.layer(l, B_QKV));
    g.ln = 1; g.ln_g = Wp(c, o.layer(l, LN1_G)); g.ln_b = Wp(c, o.layer(l, LN1_B));
    g.epi = DECODE_QKV; g.out = dl.q; g.ldo = d; g.N = 3 * d; g.K = d;
    g.kc = dl.k(l); g.vc = dl.v(l);
    TRY(decode_gemv(f32, g, st));
    TRY(decode_attention(f32, dl.k(l), dl.v(l), dl.q, dl.o, pos, batch, (int)s.H, (int)s.hd, max_len, st));
    // x += o W_o^T + b_o
    g.in = dl.o; g.in_t = 0; g.W = Wp(c, o.layer(l, W_O)); g.bias = Wp(c, o.layer(l, B_O));
    g.ln = 0; g.epi = DECODE_RESID; g.out = dl.x; g.ldo = d; g.N = d; g.K = d;
    TRY(decode_gemv(f32, g, st));
    // LN2 -> fc (+ bias) -> GELU
    g.in = dl.x; g.in_t = 0; g.W = Wp(c, o.layer(l, W_FC)); g.bias = Wp(c, o.layer(l, B_FC));
    g.ln = 1; g.ln_g = Wp(c, o.layer(l, LN2_G)); g.ln_b = Wp(c, o.layer(l, LN2_B));
    g.epi = DECODE_GELU; g.out = dl.g; g.ldo = 4 * d; g.N = 4 * d; g.K = d;  // GELU(u) in the compute dtype
    TRY(decode_gemv(f32, g, st));
    // x += g W_mp^T + b_mp
    g.in = dl.g; g.in_t = 1; g.W = Wp(c, o.layer(l, W_MP)); g.bias = Wp(c, o.layer(l, B_MP));
    g.ln = 0; g.epi = DECODE_RESID; g.out = dl.x; g.ldo = d; g.N = d; g.K = 4 * d;
    TRY(decode_gemv(f32, g, st));
  }
  // final LN -> tied LM head
  g.in = dl.x; g.in_t = 0; g.W = Wp(c, o.wte()); g.bias = nullptr;
  g.ln = 1; g.ln_g = Wp(c, o.lnf_g()); g.ln_b = Wp(c, o.lnf_b());
  g.epi = DECODE_LOGITS; g.out = logits; g.ldo = s.V; g.N = (int)s.V; g.K = d;
  return decode_gemv(f32, g, st);
}

int gpt2_prefill(gpt2_ctx* c, void* cache, size_t cache_bytes, int batch, int max_len, const int32_t* tokens,
                 const int32_t* prompt_len, float* logits, void* stream) {
  DecodeLayout dl;
  TRY(decode_check(c, cache, cache_bytes, batch, max_len, &dl));
  if (!tokens || !prompt_len || !logits) return GPT2_ERR_INVALID_ARG;
  if (batch > c->cfg.max_batch) return GPT2_ERR_INVALID_ARG;
  const Shape& s = c->s;
  if (s.mode == 0 && (batch * s.T) % 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = S(stream);
  const int f32 = s.mode;
  TRY(forward_logits(c, tokens, batch, st));
  for (int l = 0; l < (int)s.L; ++l)
    TRY(prefill_kv(f32, c->w.layers[l].qkv, dl.k(l), dl.v(l), prompt_len, batch, (int)s.T, (int)s.H, (int)s.hd,
                   max_len, max_len, c->w.err, st));
  return prefill_logits(f32, c->w.logits, prompt_len, logits, batch, (int)s.T, (int)s.V, max_len, st);
}

int gpt2_greedy_next(gpt2_ctx* c, const float* logits, int batch, int32_t* next_tokens, int32_t* pos,
                     void* stream) {
  if (!c || !logits || !next_tokens || batch < 1) return GPT2_ERR_INVALID_ARG;
  return decode_greedy(logits, c->s.V, batch, (int)c->s.Vr, next_tokens, pos, c->w.greedy_v, c->w.greedy_i,
                       S(stream));
}

int gpt2_step_host(gpt2_ctx* c, const int32_t* tokens_host, const int32_t* targets_host, int batch,
                   float* loss_host, float lr, float beta1, float beta2, float eps, float weight_decay, int step,
                   void* stream) {
  if (!c || !tokens_host || !targets_host || !loss_host) return GPT2_ERR_INVALID_ARG;
  if (batch < 1 || batch > c->cfg.max_batch) return GPT2_ERR_INVALID_ARG;
  cudaStream_t st = S(stream);
  const size_t bytes = (size_t)batch * c->s.T * 4;
  if (c->graph_exec && c->graph_batch == batch && c->graph_plain) {
    // the captured micro-step of this shape: ids straight into its inputs
    CUDA_TRY(cudaMemcpyAsync(c->w.gtok, tokens_host, bytes, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(c->w.gtgt, targets_host, bytes, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaGraphLaunch(c->graph_exec, st));
    g_launches.fetch_add(c->graph_launches, std::memory_order_relaxed);
    c->have_fwd = 1;
    c->fwd_batch = batch;
  } else {
    CUDA_TRY(cudaMemcpyAsync(c->w.tok_stage, tokens_host, bytes, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(c->w.tgt_stage, targets_host, bytes, cudaMemcpyHostToDevice, st));
    TRY(gpt2_forward_loss(c, c->w.tok_stage, c->w.tgt_stage, batch, c->w.loss, stream));
    TRY(gpt2_backward(c, 1.f, 0, stream));
  }
  TRY(gpt2_adamw_step(c, lr, beta1, beta2, eps, weight_decay, step, stream));
  const float* loss_src = (c->graph_exec && c->graph_batch == batch && c->graph_plain) ? c->graph_loss : c->w.loss;
  CUDA_TRY(cudaMemcpyAsync(loss_host, loss_src, sizeof(float), cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  return GPT2_OK;
}

uint64_t gpt2_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int gpt2_graph_release(gpt2_ctx* c) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  if (c->graph_exec) CUDA_TRY(cudaGraphExecDestroy(c->graph_exec));
  if (c->graph) CUDA_TRY(cudaGraphDestroy(c->graph));
  c->graph_exec = nullptr;
  c->graph = nullptr;
  c->graph_batch = 0;
  c->graph_plain = 0;
  c->graph_launches = 0;
  return GPT2_OK;
}

int gpt2_graph_capture(gpt2_ctx* c, int batch, float grad_scale, int accumulate, float* loss_dev, void* stream) {
  if (!c || !stream) return GPT2_ERR_INVALID_ARG;
  if (batch < 1 || batch > c->cfg.max_batch) return GPT2_ERR_INVALID_ARG;
  TRY(gpt2_graph_release(c));
  cudaStream_t st = S(stream);
  const unsigned long long l0 = g_launches.load(std::memory_order_relaxed);
  CUDA_TRY(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
  // the recorded forward reads the graph's own input buffers
  int rc = gpt2_forward_loss(c, c->w.gtok, c->w.gtgt, batch, loss_dev, stream);
  if (rc == GPT2_OK) rc = backward_impl(c, grad_scale, accumulate, nullptr, stream);
  cudaGraph_t g = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(st, &g);
  const unsigned long long n = g_launches.load(std::memory_order_relaxed) - l0;
  // the capture launched nothing: take its kernels back out of the count
  g_launches.fetch_sub(n, std::memory_order_relaxed);
  c->have_fwd = 0;
  if (rc != GPT2_OK || ec != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return rc != GPT2_OK ? rc : GPT2_ERR_CUDA;
  }
  cudaGraphExec_t ex = nullptr;
  if (cudaGraphInstantiate(&ex, g, 0) != cudaSuccess) {
    cudaGraphDestroy(g);
    cudaGetLastError();
    return GPT2_ERR_CUDA;
  }
  c->graph = g;
  c->graph_exec = ex;
  c->graph_batch = batch;
  c->graph_plain = (grad_scale == 1.f && accumulate == 0) ? 1 : 0;
  c->graph_loss = loss_dev ? loss_dev : c->w.loss;
  c->graph_launches = n;
  return GPT2_OK;
}

int gpt2_graph_step(gpt2_ctx* c, const int32_t* tokens, const int32_t* targets, void* stream) {
  if (!c || !tokens || !targets) return GPT2_ERR_INVALID_ARG;
  if (!c->graph_exec) return GPT2_ERR_BAD_STATE;
  cudaStream_t st = S(stream);
  const size_t bytes = (size_t)c->graph_batch * c->s.T * 4;
  CUDA_TRY(cudaMemcpyAsync(c->w.gtok, tokens, bytes, cudaMemcpyDeviceToDevice, st));
  CUDA_TRY(cudaMemcpyAsync(c->w.gtgt, targets, bytes, cudaMemcpyDeviceToDevice, st));
  CUDA_TRY(cudaGraphLaunch(c->graph_exec, st));
  g_launches.fetch_add(c->graph_launches, std::memory_order_relaxed);
  // as after gpt2_forward_loss + gpt2_backward
  c->have_fwd = 1;
  c->fwd_batch = c->graph_batch;
  return GPT2_OK;
}

const char* gpt2_strerror(int code) {
  switch (code) {
    case GPT2_OK: return "ok";
    case GPT2_ERR_INVALID_ARG: return "invalid argument";
    case GPT2_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case GPT2_ERR_CUDA: return "CUDA error";
    case GPT2_ERR_BAD_STATE: return "bad state (backward without forward?)";
    case GPT2_ERR_TOKEN_RANGE: return "token or target id out of range";
    case GPT2_ERR_NONFINITE: return "non-finite loss";
    case GPT2_ERR_TIMEOUT: return "device pipeline wait timed out";
    case GPT2_ERR_WORKSPACE: return "workspace too small";
    case GPT2_ERR_TOO_LARGE: return "problem exceeds the built-in scratch of the allocation-free entry point";
    case GPT2_ERR_POSITION_RANGE: return "decode position or prompt length out of range";
    default: return "unknown error";
  }
}

int gpt2_op_gemm_bf16(const uint16_t* A, int a_mn_major, int lda, const uint16_t* B, int b_mn_major, int ldb,
                      void* C, int c_fp32, int ldc, int M, int N, int K, float alpha, float beta, void* workspace,
                      size_t workspace_bytes, int bn, int splits, void* stream) {
  if (!A || !B || !C || M < 0 || N < 0 || K < 0) return GPT2_ERR_INVALID_ARG;
  GemmArgs g = make_gemm(M, N, K, A, a_mn_major ? 1 : 0, lda, B, b_mn_major ? 1 : 0, ldb,
                         c_fp32 ? EPI_F32 : EPI_STORE, C, ldc);
  g.epi.alpha = alpha;
  g.epi.beta = c_fp32 ? beta : 0.f;
  return gemm_tc_bf16(g, workspace, workspace_bytes, bn, splits, nullptr, S(stream));
}

int gpt2_op_linear_bf16(const uint16_t* x, const uint16_t* w, const uint16_t* bias, const uint16_t* resid,
                        uint16_t* out, uint16_t* out2, int M, int N, int K, int act, void* stream) {
  if (!x || !w || !bias || !out || M < 0 || N < 0 || K < 0 || act < 0 || act > 2) return GPT2_ERR_INVALID_ARG;
  if ((act == 1 && !resid) || (act == 2 && !out2)) return GPT2_ERR_INVALID_ARG;
  const uintptr_t al = (uintptr_t)x | (uintptr_t)w | (uintptr_t)bias | (uintptr_t)out |
                       (act == 1 ? (uintptr_t)resid : 0) | (act == 2 ? (uintptr_t)out2 : 0);
  if (al & 15) return GPT2_ERR_INVALID_ARG;
  if (K % 64 || N % 8) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return GPT2_OK;
  static const int kinds[3] = {EPI_BIAS, EPI_BIAS_RESID, EPI_BIAS_GELU};
  // the GELU epilogue writes GELU'(u) to epi.out and GELU(u) to epi.out2
  GemmArgs g = make_gemm(M, N, K, x, 0, K, w, 0, K, kinds[act], act == 2 ? (void*)out2 : (void*)out, N);
  g.epi.bias = bias;
  if (act == 1) g.epi.resid = resid;
  if (act == 2) g.epi.out2 = out;
  return gemm_tc_bf16(g, nullptr, 0, 0, 1, nullptr, S(stream));
}

int gpt2_set_wait_timeout_ns(uint64_t ns) {
  const unsigned long long v = ns ? (unsigned long long)ns : WAIT_TIMEOUT_NS;
  TRY(gemm_tc_set_wait_limit(v));
  return attn_tc_set_wait_limit(v);
}

int gpt2_op_gemm_bf16_status(const uint16_t* A, int a_mn_major, int lda, const uint16_t* B, int b_mn_major, int ldb,
                             void* C, int c_fp32, int ldc, int M, int N, int K, float alpha, float beta,
                             void* workspace, size_t workspace_bytes, int bn, int splits, int* status,
                             void* stream) {
  if (!A || !B || !C || !status || M < 0 || N < 0 || K < 0) return GPT2_ERR_INVALID_ARG;
  if ((uintptr_t)status & 3) return GPT2_ERR_INVALID_ARG;
  GemmArgs g = make_gemm(M, N, K, A, a_mn_major ? 1 : 0, lda, B, b_mn_major ? 1 : 0, ldb,
                         c_fp32 ? EPI_F32 : EPI_STORE, C, ldc);
  g.epi.alpha = alpha;
  g.epi.beta = c_fp32 ? beta : 0.f;
  return gemm_tc_bf16(g, workspace, workspace_bytes, bn, splits, status, S(stream));
}

int gpt2_op_attention_fwd_bf16(const uint16_t* qkv, uint16_t* o, float* lse, int B, int T, int H, int hd,
                               void* stream) {
  if (!qkv || !o || !lse || B < 0 || T < 0 || H < 1) return GPT2_ERR_INVALID_ARG;
  return attn_fwd_bf16(qkv, o, lse, B, T, H, hd, S(stream));
}

int gpt2_op_attention_bwd_bf16(const uint16_t* qkv, const uint16_t* o, const float* lse, const uint16_t* dout,
                               uint16_t* dqkv, float* scratch, int B, int T, int H, int hd, void* stream) {
  if (!qkv || !o || !lse || !dout || !dqkv || !scratch || B < 0 || T < 0 || H < 1) return GPT2_ERR_INVALID_ARG;
  float* dq_acc = scratch;
  float* dvec = scratch + (size_t)B * T * H * hd;
  return attn_bwd_bf16(qkv, o, lse, dout, dqkv, dq_acc, dvec, B, T, H, hd, S(stream));
}

// ---- single HBM-bound steps of the path (kernel tests and profiling) ----

int gpt2_op_layernorm_fwd_bf16(const uint16_t* x, const uint16_t* gamma, const uint16_t* beta, uint16_t* y,
                               float* mean, float* rstd, int M, int d, void* stream) {
  if (!x || !gamma || !beta || !y || !mean || !rstd || M < 0 || d < 1) return GPT2_ERR_INVALID_ARG;
  if (d % 64 || d > 2048) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (((uintptr_t)x | (uintptr_t)y | (uintptr_t)gamma | (uintptr_t)beta) & 15) return GPT2_ERR_INVALID_ARG;
  if (M == 0) return GPT2_OK;
  return layernorm_fwd(0, x, gamma, beta, y, mean, rstd, M, d, S(stream));
}

size_t gpt2_op_layernorm_bwd_scratch_floats(int M, int d) {
  if (M < 1 || d < 1) return 0;
  return layernorm_bwd_part_floats(M, d);
}

int gpt2_op_layernorm_bwd_bf16(const uint16_t* dy, const uint16_t* x, const float* mean, const float* rstd,
                               const uint16_t* gamma, uint16_t* dx, int accumulate, float* dgamma_dbeta,
                               float* scratch, size_t scratch_floats, int M, int d, void* stream) {
  if (!dy || !x || !mean || !rstd || !gamma || !dx || !dgamma_dbeta || !scratch || M < 1 || d < 1)
    return GPT2_ERR_INVALID_ARG;
  if (d % 64 || d > 2048) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (((uintptr_t)dy | (uintptr_t)x | (uintptr_t)dx | (uintptr_t)gamma | (uintptr_t)scratch) & 15)
    return GPT2_ERR_INVALID_ARG;
  if (scratch_floats < layernorm_bwd_part_floats(M, d)) return GPT2_ERR_WORKSPACE;
  const cudaStream_t st = S(stream);
  int nblk = 0;
  TRY(layernorm_bwd(0, dy, x, mean, rstd, gamma, dx, accumulate ? 0 : 1, scratch, nullptr, &nblk, M, d, st));
  return reduce_rows_f32(scratch, nblk, 2 * d, dgamma_dbeta, 0.f, st);
}

size_t gpt2_op_colsum_scratch_floats(int M, int N) {
  if (M < 1 || N < 1) return 0;
  return colsum_part_floats(M, N);
}

int gpt2_op_colsum_bf16(const uint16_t* x, int M, int N, float* out, float* scratch, size_t scratch_floats,
                        void* stream) {
  if (!x || !out || !scratch || M < 1 || N < 1) return GPT2_ERR_INVALID_ARG;
  if (N % 8 || ((uintptr_t)x & 15)) return GPT2_ERR_INVALID_ARG;
  if (scratch_floats < colsum_part_floats(M, N)) return GPT2_ERR_WORKSPACE;
  const cudaStream_t st = S(stream);
  int nblk = 0;
  TRY(colsum_partial(0, x, M, N, scratch, &nblk, st));
  return reduce_rows_f32(scratch, nblk, N, out, 0.f, st);
}

// ---- the LM head with its fused softmax cross-entropy, alone --------------

namespace {
// Scratch of the LM-head cross-entropy ops: status word, n_valid, then the
// bf16 [M, V] buffer (the forward's exponentials, rewritten as dz), the
// per-part maxima and sums [V/128][M], the target logits and the row
// log-sum-exps [M].
struct CeScratch {
  int* err;
  int* n_valid;
  void* e;
  float *pm, *ps, *zt, *lse;
  size_t bytes;
};
CeScratch ce_scratch(void* base, int M, int V) {
  Carver c{(uint8_t*)base};
  CeScratch s;
  s.err = c.take<int>(4);
  s.n_valid = c.take<int>(4);
  s.e = c.take<void>((size_t)M * V * 2);
  s.pm = c.take<float>((size_t)(V / 128) * M * 4);
  s.ps = c.take<float>((size_t)(V / 128) * M * 4);
  s.zt = c.take<float>((size_t)M * 4);
  s.lse = c.take<float>((size_t)M * 4);
  s.bytes = (c.off + 255) & ~(size_t)255;
  return s;
}
}  // namespace

size_t gpt2_op_lm_head_ce_scratch_bytes(int M, int V) {
  if (M < 1 || V < 128 || V % 128) return 0;
  return ce_scratch(nullptr, M, V).bytes;
}

int gpt2_op_lm_head_ce_fwd_bf16(const uint16_t* x, const uint16_t* w, const int32_t* targets, int M, int V, int d,
                                int vocab_real, float* loss, float* loss_rows, void* scratch, size_t scratch_bytes,
                                void* stream) {
  if (!x || !w || !targets || !loss || !loss_rows || !scratch || M < 1 || d < 1) return GPT2_ERR_INVALID_ARG;
  if (V < 128 || V % 128 || d % 64 || vocab_real < 1 || vocab_real > V) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (((uintptr_t)x | (uintptr_t)w | (uintptr_t)scratch) & 255) return GPT2_ERR_INVALID_ARG;
  const CeScratch cs = ce_scratch(scratch, M, V);
  if (scratch_bytes < cs.bytes) return GPT2_ERR_WORKSPACE;
  const cudaStream_t st = S(stream);
  CUDA_TRY(cudaMemsetAsync(cs.err, 0, sizeof(int), st));
  GemmArgs g = make_gemm(M, V, d, x, 0, d, w, 0, d, EPI_CE_FWD, cs.e, V);
  g.epi.ce_max = cs.pm;
  g.epi.ce_sum = cs.ps;
  g.epi.ce_zt = cs.zt;
  g.epi.ce_tgt = targets;
  TRY(gemm_tc_bf16(g, nullptr, 0, 0, 1, cs.err, st));
  TRY(count_targets(targets, M, vocab_real, cs.n_valid, cs.err, st));
  TRY(ce_merge_dz(cs.pm, cs.ps, cs.zt, targets, cs.e, cs.lse, M, V, vocab_real, cs.n_valid, loss_rows, st));
  return loss_mean(loss_rows, M, cs.n_valid, loss, cs.err, st);
}

int gpt2_op_lm_head_ce_bwd_bf16(const uint16_t* x, const uint16_t* w, int M, int V, int d, float grad_scale,
                                uint16_t* dx, float* dw, int accumulate, void* scratch, size_t scratch_bytes,
                                void* stream) {
  if (!x || !w || !dx || !dw || !scratch || M < 1 || d < 1) return GPT2_ERR_INVALID_ARG;
  if (V < 128 || V % 128 || d % 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  if (((uintptr_t)x | (uintptr_t)w | (uintptr_t)dx | (uintptr_t)dw | (uintptr_t)scratch) & 255)
    return GPT2_ERR_INVALID_ARG;
  const CeScratch cs = ce_scratch(scratch, M, V);
  if (scratch_bytes < cs.bytes) return GPT2_ERR_WORKSPACE;
  const cudaStream_t st = S(stream);
  GemmArgs g = make_gemm(M, d, V, cs.e, 0, V, w, 1, d, EPI_STORE, dx, d);
  g.epi.alpha = grad_scale / (float)M;
  TRY(gemm_tc_bf16(g, nullptr, 0, 0, 1, cs.err, st));
  g = make_gemm(V, d, M, cs.e, 1, V, x, 1, d, EPI_F32, dw, d);
  g.epi.alpha = grad_scale / (float)M;
  g.epi.beta = accumulate ? 1.f : 0.f;
  return gemm_tc_bf16(g, nullptr, 0, 0, 1, cs.err, st);
}

}  // extern "C"
