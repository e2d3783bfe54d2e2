#include <stdlib.h>
// GPT-2 training step behind the C ABI of gpt2_b200.h: owns the parameters (fp32 master
// weights in one flat buffer, canonical order), their bf16 copies, the gradients, the
// AdamW moments and the activation arena, and enqueues the kernels of one forward,
// backward and optimizer step on one CUDA stream.
//
// The schedule follows GPT.forward / Block.forward / CausalSelfAttention.forward and the
// training loop of "Karpathy's Zero to Hero, Lecture 9: Reproduce GPT-2 (124M)" notes
// (section "Code you'll write"), with the backward of each op written out.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "gpt2_b200.h"
#include "common.cuh"
#include "gemm.h"
#include "kernels.h"

namespace {

enum ProfClass {
  PROF_GEMM_FWD = GPT2_PROF_GEMM_FWD, PROF_GEMM_BWD = GPT2_PROF_GEMM_BWD, PROF_HEAD_FWD = GPT2_PROF_HEAD_FWD,
  PROF_HEAD_BWD = GPT2_PROF_HEAD_BWD, PROF_ATTN_FWD = GPT2_PROF_ATTN_FWD, PROF_ATTN_BWD = GPT2_PROF_ATTN_BWD,
  PROF_LN_FWD = GPT2_PROF_LN_FWD, PROF_LN_BWD = GPT2_PROF_LN_BWD, PROF_CE = GPT2_PROF_CE, PROF_BIAS = GPT2_PROF_BIAS,
  PROF_EMBED = GPT2_PROF_EMBED, PROF_OPTIM = GPT2_PROF_OPTIM
};

enum LayerParam {
  LN1_W = 0, LN1_B, ATTN_W, ATTN_B, PROJ_W, PROJ_B, LN2_W, LN2_B, FC_W, FC_B, MPROJ_W, MPROJ_B, NLP
};

struct ParamView {
  long long off, n;
  int decay;
  double std;   // < 0: constant init (value in `fill`)
  float fill;
};

struct LayerActs {
  void* ln1;
  float* ln1_mean;
  float* ln1_rstd;
  void* qkv;
  void* attn;
  float* attn_lse;
  float* x1;
  void* ln2;
  float* ln2_mean;
  float* ln2_rstd;
  void* fc_pre;     // gelu'(u) of the fc pre-activation u, kept for the backward
  void* fc_act;
};

uint64_t splitmix64_host(uint64_t state, uint64_t j) {
  uint64_t z = state + (j + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

}  // namespace

struct gpt2_ctx {
  gpt2_config cfg;
  bool bf16 = false;
  int num_sms = 148;
  int device = 0;
  cudaStream_t stream = nullptr;
  cudaStream_t own_stream = nullptr;
  std::string err;
  std::vector<void*> allocs;

  long long nparams = 0;
  std::vector<ParamView> views;
  float* params = nullptr;
  float* grads = nullptr;
  float* m = nullptr;
  float* v = nullptr;
  uint16_t* shadow = nullptr;
  AdamBlock* adam_blocks = nullptr;
  int n_adam_blocks = 0;
  long long step_t = 0;

  int Nmax = 0;
  size_t act = 4;   // bytes per activation element
  std::vector<LayerActs> layers;
  float* resid = nullptr;   // [(L+1) * Nmax * C]
  void* lnf = nullptr;
  float* lnf_mean = nullptr;
  float* lnf_rstd = nullptr;
  void* logits = nullptr;
  long long ldl = 0;
  CePartial* ce_part = nullptr;
  float* zt = nullptr;
  float* lse = nullptr;
  float* loss_row = nullptr;
  int* argmax = nullptr;
  float* scalars = nullptr;   // [0] loss [1] dz scale [2] grad norm [3] clip scale
  int* count = nullptr;
  int* tokens = nullptr;
  int* targets = nullptr;

  float* dres = nullptr;
  void* dres_act = nullptr;
  void* dy = nullptr;       // gradient of a LayerNorm output (activation type)
  void* d4c = nullptr;
  void* dqkv = nullptr;
  void* dattn = nullptr;
  float* attnD = nullptr;
  // Partial column sums that the backward leaves behind and one batched launch at its end
  // reduces: per layer, the c_attn bias sums from the attention backward and the c_fc bias
  // sums per 32 rows from the c_proj dX GEMM; per LayerNorm (ln_1 and ln_2 of each layer, then
  // ln_f), the weight, bias and upstream Linear bias sums per LayerNorm backward block.
  float* attn_bias_part = nullptr;
  size_t attn_bias_stride = 0;
  float* fc_bias_part = nullptr;
  size_t fc_bias_stride = 0;
  float* ln_part = nullptr;
  int ln_blocks = 0;
  float* colsum_part = nullptr;
  uint64_t* enc_sorted = nullptr;
  uint32_t* enc_seg = nullptr;
  float* enc_part = nullptr;
  float* splitk_ws = nullptr;
  size_t splitk_ws_elems = 0;
  double* norm_part = nullptr;
  int norm_nparts = 0;

  int lastB = 0, lastT = 0;
  // CUDA graphs of the forward / backward launch sequences, one per (kind, B, T): the first
  // call with a key runs eagerly, the second is captured, later ones replay the graph
  struct GraphEntry {
    int kind, B, T, calls;
    cudaGraphExec_t exec;
    long long launches;
  };
  std::vector<GraphEntry> graphs;
  bool use_graphs = true;
  bool have_targets = false;
  bool have_logits = false;   // the last forward's logits are intact (no backward since)

  // per-kernel-class CUDA-event profiling (gpt2_profile_start / gpt2_profile_stop)
  bool prof_on = false;
  std::vector<cudaEvent_t> prof_events;
  size_t prof_used = 0;
  std::vector<int> prof_class;          // class of event pair i
  double prof_flops[GPT2_PROF_CLASSES] = {0};
  double prof_bytes[GPT2_PROF_CLASSES] = {0};
  long long prof_launches[GPT2_PROF_CLASSES] = {0};
};

namespace {

int fail(gpt2_ctx* c, int code, const char* msg) {
  if (c) c->err = msg;
  return code;
}

int cuda_fail(gpt2_ctx* c, cudaError_t e, const char* where) {
  if (c) c->err = std::string(where) + ": " + cudaGetErrorString(e);
  return GPT2_ERR_CUDA;
}

// Host-to-device copy ordered on the context stream and complete on return.  A plain
// cudaMemcpy from pageable host memory may return before its DMA has landed, and runs on the
// legacy default stream, which does not order against the context's non-blocking stream: a
// kernel launched right after could read the old contents.
cudaError_t h2d_ordered(gpt2_ctx* c, void* dst, const void* src, size_t bytes) {
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, c->stream);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(c->stream);
}

template <typename T>
int dalloc(gpt2_ctx* c, T** p, size_t count) {
  void* q = nullptr;
  if (count == 0) count = 1;
  cudaError_t e = cudaMalloc(&q, count * sizeof(T));
  if (e != cudaSuccess) {
    c->err = "device allocation failed";
    return GPT2_ERR_OOM;
  }
  c->allocs.push_back(q);
  *p = reinterpret_cast<T*>(q);
  return GPT2_OK;
}
int dalloc_bytes(gpt2_ctx* c, void** p, size_t bytes) {
  char* q = nullptr;
  int rc = dalloc<char>(c, &q, bytes);
  *p = q;
  return rc;
}

int param_index(const gpt2_config& cfg, int layer, int p) { return 2 + NLP * layer + p; }
int lnf_w_index(const gpt2_config& cfg) { return 2 + NLP * cfg.n_layer; }

float* P(gpt2_ctx* c, int idx) { return c->params + c->views[idx].off; }
float* G(gpt2_ctx* c, int idx) { return c->grads + c->views[idx].off; }
// GEMM weight operand: the bf16 copy in bf16 mode, the fp32 master in fp32 mode.
const void* W(gpt2_ctx* c, int idx) {
  if (c->bf16) return c->shadow + c->views[idx].off;
  return c->params + c->views[idx].off;
}

int build_views(gpt2_ctx* c) {
  const gpt2_config& g = c->cfg;
  const long long C = g.n_embd, Vp = g.padded_vocab_size, T = g.block_size;
  const double s0 = 0.02, sres = 0.02 / std::sqrt(2.0 * g.n_layer);
  long long off = 0;
  auto add = [&](long long n, int decay, double std, float fill) {
    ParamView v;
    v.off = off;
    v.n = n;
    v.decay = decay;
    v.std = std;
    v.fill = fill;
    c->views.push_back(v);
    off += n;
  };
  add(Vp * C, 1, s0, 0.f);   // wte
  add(T * C, 1, s0, 0.f);    // wpe
  for (int l = 0; l < g.n_layer; ++l) {
    add(C, 0, -1, 1.f);            // ln_1.weight
    add(C, 0, -1, 0.f);            // ln_1.bias
    add(3 * C * C, 1, s0, 0.f);    // attn.c_attn.weight
    add(3 * C, 0, -1, 0.f);        // attn.c_attn.bias
    add(C * C, 1, sres, 0.f);      // attn.c_proj.weight
    add(C, 0, -1, 0.f);            // attn.c_proj.bias
    add(C, 0, -1, 1.f);            // ln_2.weight
    add(C, 0, -1, 0.f);            // ln_2.bias
    add(4 * C * C, 1, s0, 0.f);    // mlp.c_fc.weight
    add(4 * C, 0, -1, 0.f);        // mlp.c_fc.bias
    add(4 * C * C, 1, sres, 0.f);  // mlp.c_proj.weight
    add(C, 0, -1, 0.f);            // mlp.c_proj.bias
  }
  add(C, 0, -1, 1.f);   // ln_f.weight
  add(C, 0, -1, 0.f);   // ln_f.bias
  c->nparams = off;
  return GPT2_OK;
}

int gemm(gpt2_ctx* c, int M, int N, int K, const void* A, long long lda, bool a_mn, const void* B, long long ldb,
         bool b_mn, const EpiParams& ep) {
  int rc;
  if (c->bf16)
    rc = gemm_bf16_tc(c->stream, M, N, K, A, lda, a_mn, B, ldb, b_mn, ep, c->splitk_ws, c->splitk_ws_elems,
                      c->num_sms);
  else
    rc = gemm_f32_simt(c->stream, M, N, K, reinterpret_cast<const float*>(A), lda, a_mn,
                       reinterpret_cast<const float*>(B), ldb, b_mn, ep);
  if (rc) c->err = "gemm launch failed";
  return rc;
}

int check_device(gpt2_ctx* c) {
  cudaError_t e = cudaStreamSynchronize(c->stream);
  if (e != cudaSuccess) return cuda_fail(c, e, "stream synchronize");
  int code = 0;
  if (read_and_clear_device_error(&code)) return fail(c, GPT2_ERR_CUDA, "reading the device error word failed");
  switch (code) {
    case DEVERR_NONE: return GPT2_OK;
    case DEVERR_TOKEN: return fail(c, GPT2_ERR_TOKEN, "input token id outside [0, vocab_size)");
    case DEVERR_TARGET: return fail(c, GPT2_ERR_TARGET, "target outside [0, vocab_size) and not -1");
    case DEVERR_TIMEOUT: return fail(c, GPT2_ERR_TIMEOUT, "a bounded device wait timed out");
    case DEVERR_ROW: return fail(c, GPT2_ERR_ARG, "a sampled row outside the last forward's B*T rows");
    default: return fail(c, GPT2_ERR_CUDA, "device reported an internal error");
  }
}

// Brackets one launch (or a short group of launches) of kernel class `cls` with a pair of
// events on the context stream while profiling is on.
struct ProfScope {
  gpt2_ctx* c;
  int cls;
  ProfScope(gpt2_ctx* c_, int cls_, double flops, double bytes) : c(c_), cls(cls_) {
    if (!c->prof_on) return;
    c->prof_flops[cls] += flops;
    c->prof_bytes[cls] += bytes;
    c->prof_launches[cls] += 1;
    if (c->prof_used + 2 > c->prof_events.size()) {
      for (int i = 0; i < 256; ++i) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) break;
        c->prof_events.push_back(e);
      }
    }
    if (c->prof_used + 2 <= c->prof_events.size()) cudaEventRecord(c->prof_events[c->prof_used], c->stream);
  }
  ~ProfScope() {
    if (!c->prof_on) return;
    if (c->prof_used + 2 <= c->prof_events.size()) {
      cudaEventRecord(c->prof_events[c->prof_used + 1], c->stream);
      c->prof_used += 2;
      c->prof_class.push_back(cls);
    }
  }
};

#define RC(x)                 \
  do {                        \
    int _r = (x);             \
    if (_r != 0) return _r;   \
  } while (0)

#define PROF(cls, flops, bytes) ProfScope _prof_scope_(c, (cls), (double)(flops), (double)(bytes))

int forward_impl(gpt2_ctx* c, int B, int T, bool with_targets) {
  const gpt2_config& g = c->cfg;
  const int N = B * T, C = g.n_embd, H = g.n_head, hd = C / H, L = g.n_layer, Vp = g.padded_vocab_size;
  const double Nd = N, Cd = C, A = (double)c->act;
  cudaStream_t st = c->stream;
  {
    PROF(PROF_EMBED, 0, 8.0 * Nd * Cd + 4.0 * T * Cd);
    RC(launch_encoder_fwd(st, c->tokens, P(c, 0), P(c, 1), c->resid, N, T, C, g.vocab_size));
  }
  const double ln_fwd_bytes = Nd * Cd * (4.0 + A) + 8.0 * Nd;
  for (int l = 0; l < L; ++l) {
    LayerActs& a = c->layers[l];
    float* x = c->resid + (long long)l * c->Nmax * C;
    float* xo = c->resid + (long long)(l + 1) * c->Nmax * C;
    auto pi = [&](int p) { return param_index(g, l, p); };
    // x = x + attn(ln_1(x))
    {
      PROF(PROF_LN_FWD, 0, ln_fwd_bytes);
      RC(launch_layernorm_fwd(st, c->bf16, x, P(c, pi(LN1_W)), P(c, pi(LN1_B)), a.ln1, a.ln1_mean, a.ln1_rstd, N,
                              C));
    }
    EpiParams e = epi_make(EPI_STORE_ACT, a.qkv, 3 * C);
    e.bias = P(c, pi(ATTN_B));
    {
      PROF(PROF_GEMM_FWD, 2.0 * Nd * 3 * Cd * Cd, 0);
      RC(gemm(c, N, 3 * C, C, a.ln1, C, false, W(c, pi(ATTN_W)), C, false, e));
    }
    {
      PROF(PROF_ATTN_FWD, 2.0 * B * (double)T * T * Cd, 0);
      RC(launch_attn_fwd(st, c->bf16, a.qkv, a.attn, a.attn_lse, B, T, H, hd));
    }
    e = epi_make(EPI_RESID_F32, a.x1, C);
    e.bias = P(c, pi(PROJ_B));
    e.aux = x;
    e.ld_aux = C;
    {
      PROF(PROF_GEMM_FWD, 2.0 * Nd * Cd * Cd, 0);
      RC(gemm(c, N, C, C, a.attn, C, false, W(c, pi(PROJ_W)), C, false, e));
    }
    // x = x + mlp(ln_2(x))
    {
      PROF(PROF_LN_FWD, 0, ln_fwd_bytes);
      RC(launch_layernorm_fwd(st, c->bf16, a.x1, P(c, pi(LN2_W)), P(c, pi(LN2_B)), a.ln2, a.ln2_mean, a.ln2_rstd,
                              N, C));
    }
    e = epi_make(EPI_GELU_FWD, a.fc_act, 4 * C);
    e.bias = P(c, pi(FC_B));
    e.aux_out = a.fc_pre;
    e.ld_aux_out = 4 * C;
    {
      PROF(PROF_GEMM_FWD, 2.0 * Nd * 4 * Cd * Cd, 0);
      RC(gemm(c, N, 4 * C, C, a.ln2, C, false, W(c, pi(FC_W)), C, false, e));
    }
    e = epi_make(EPI_RESID_F32, xo, C);
    e.bias = P(c, pi(MPROJ_B));
    e.aux = a.x1;
    e.ld_aux = C;
    {
      PROF(PROF_GEMM_FWD, 2.0 * Nd * 4 * Cd * Cd, 0);
      RC(gemm(c, N, C, 4 * C, a.fc_act, 4 * C, false, W(c, pi(MPROJ_W)), 4 * C, false, e));
    }
  }
  const int lf = lnf_w_index(g);
  float* xL = c->resid + (long long)L * c->Nmax * C;
  {
    PROF(PROF_LN_FWD, 0, ln_fwd_bytes);
    RC(launch_layernorm_fwd(st, c->bf16, xL, P(c, lf), P(c, lf + 1), c->lnf, c->lnf_mean, c->lnf_rstd, N, C));
  }
  // tied lm_head: logits = ln_f(x) wte^T
  const double head_flops = 2.0 * Nd * Vp * Cd;
  if (c->bf16) {
    EpiParams e = epi_make(with_targets ? EPI_CE_FWD : EPI_STORE_ACT, c->logits, c->ldl);
    if (with_targets) {
      e.targets = c->targets;
      e.ce_part = c->ce_part;
      e.zt = c->zt;
    }
    {
      PROF(PROF_HEAD_FWD, head_flops, 0);
      RC(gemm(c, N, Vp, C, c->lnf, C, false, W(c, 0), C, false, e));
    }
    if (with_targets) {
      const int ntiles = gemm_tc_ce_tiles(Vp);
      PROF(PROF_CE, 0, 16.0 * Nd * ntiles + 16.0 * Nd);
      RC(launch_ce_finalize(st, c->ce_part, ntiles, c->zt, c->targets, N, g.vocab_size, c->lse, c->loss_row,
                            c->argmax));
    }
  } else {
    EpiParams e = epi_make(EPI_STORE_F32, c->logits, c->ldl);
    {
      PROF(PROF_HEAD_FWD, head_flops, 0);
      RC(gemm(c, N, Vp, C, c->lnf, C, false, W(c, 0), C, false, e));
    }
    if (with_targets) {
      PROF(PROF_CE, 0, 4.0 * Nd * Vp);
      RC(launch_ce_rowwise(st, reinterpret_cast<const float*>(c->logits), c->ldl, c->targets, N, Vp, g.vocab_size,
                           c->lse, c->loss_row, c->argmax));
    }
  }
  if (with_targets) {
    PROF(PROF_CE, 0, 8.0 * Nd);
    RC(launch_loss_reduce(st, c->loss_row, c->targets, N, 1.0f / (float)g.grad_accum_steps, &c->scalars[0],
                          &c->scalars[1], c->count));
  }
  return GPT2_OK;
}

int backward_impl(gpt2_ctx* c) {
  const gpt2_config& g = c->cfg;
  const int B = c->lastB, T = c->lastT;
  const int N = B * T, C = g.n_embd, H = g.n_head, hd = C / H, L = g.n_layer, Vp = g.padded_vocab_size;
  const double Nd = N, Cd = C, A = (double)c->act;
  cudaStream_t st = c->stream;
  // dlogits in place: (softmax - onehot) / (count * k)
  {
    PROF(PROF_CE, 0, 2.0 * Nd * Vp * A + 12.0 * Nd);
    RC(launch_ce_dz(st, c->bf16, c->logits, c->ldl, c->lse, c->targets, &c->scalars[1], N, Vp));
  }
  // dh = dz wte ; dwte += dz^T h
  const double head_flops = 2.0 * Nd * Vp * Cd;
  // the dX products write the LayerNorm output gradient in the activation type (bf16 in bf16 mode)
  const int dy_kind = c->bf16 ? EPI_STORE_ACT : EPI_STORE_F32;
  EpiParams e = epi_make(dy_kind, c->dy, C);
  {
    PROF(PROF_HEAD_BWD, head_flops, 0);
    RC(gemm(c, N, C, Vp, c->logits, c->ldl, false, W(c, 0), C, true, e));
  }
  e = epi_make(EPI_ACCUM_F32, G(c, 0), C);
  {
    PROF(PROF_HEAD_BWD, head_flops, 0);
    RC(gemm(c, Vp, C, N, c->logits, c->ldl, true, c->lnf, C, true, e));
  }
  const int lf = lnf_w_index(g);
  float* xL = c->resid + (long long)L * c->Nmax * C;
  const double ln_bwd_bytes = Nd * Cd * (4.0 * 3 + 2.0 * A) + 8.0 * Nd;   // dy, x, dres in; dres, dres_act out
  // the parameter and bias gradients whose partial rows are reduced in one launch at the end
  std::vector<ColsumJob> jobs;
  jobs.reserve(8 * L + 3);
  const size_t ln_slot = (size_t)c->ln_blocks * 3 * C;
  // LayerNorm partial row: [dy * xhat | dy | new dres]; the last third is the bias gradient of
  // the Linear layer that writes the residual stream there (null: none)
  auto ln_jobs = [&](const float* part, float* dw, float* db, float* dbias) {
    jobs.push_back(ColsumJob{part, dw, 3 * C, c->ln_blocks, C});
    jobs.push_back(ColsumJob{part + C, db, 3 * C, c->ln_blocks, C});
    if (dbias) jobs.push_back(ColsumJob{part + 2 * C, dbias, 3 * C, c->ln_blocks, C});
  };
  {
    PROF(PROF_LN_BWD, 0, ln_bwd_bytes - 4.0 * Nd * Cd);
    // the new dres is d loss / d x_L: its column sums are the last mlp.c_proj bias gradient
    float* part = c->ln_part + 2 * L * ln_slot;
    RC(launch_layernorm_bwd(st, c->bf16, c->dy, xL, c->lnf_mean, c->lnf_rstd, P(c, lf), c->dres, c->dres_act, false,
                            part, c->ln_blocks, N, C));
    ln_jobs(part, G(c, lf), G(c, lf + 1), G(c, param_index(g, L - 1, MPROJ_B)));
  }
  const int ncs = colsum_chunks(N);
  for (int l = L - 1; l >= 0; --l) {
    LayerActs& a = c->layers[l];
    float* x = c->resid + (long long)l * c->Nmax * C;
    auto pi = [&](int p) { return param_index(g, l, p); };
    // ---- MLP: x_out = x1 + gelu(ln2 Wfc^T + bfc) Wmp^T + bmp
    e = epi_make(EPI_ACCUM_F32, G(c, pi(MPROJ_W)), 4 * C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * 4 * Cd * Cd, 0);
      RC(gemm(c, C, 4 * C, N, c->dres_act, C, true, a.fc_act, 4 * C, true, e));
    }
    e = epi_make(EPI_GELU_BWD, c->d4c, 4 * C);
    e.aux = a.fc_pre;
    e.ld_aux = 4 * C;
    // the tensor-core path also leaves the column sums of d4C (the c_fc bias gradient) per
    // 32-row group, so d4C is not read again for them
    const bool fused_fc_bias = c->bf16 && c->fc_bias_part != nullptr;
    float* fc_part = fused_fc_bias ? c->fc_bias_part + l * c->fc_bias_stride : nullptr;
    if (fused_fc_bias) e.colsum_part = fc_part;
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * 4 * Cd * Cd, 0);
      RC(gemm(c, N, 4 * C, C, c->dres_act, C, false, W(c, pi(MPROJ_W)), 4 * C, true, e));
    }
    e = epi_make(EPI_ACCUM_F32, G(c, pi(FC_W)), C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * 4 * Cd * Cd, 0);
      RC(gemm(c, 4 * C, C, N, c->d4c, 4 * C, true, a.ln2, C, true, e));
    }
    if (fused_fc_bias) {
      jobs.push_back(ColsumJob{fc_part, G(c, pi(FC_B)), 4 * C, cdiv(N, 32), 4 * C});
    } else {
      PROF(PROF_BIAS, 0, A * Nd * 4 * Cd);
      RC(launch_colsum(st, c->bf16, c->d4c, 4 * C, N, 4 * C, c->colsum_part, ncs, G(c, pi(FC_B))));
    }
    e = epi_make(dy_kind, c->dy, C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * 4 * Cd * Cd, 0);
      RC(gemm(c, N, C, 4 * C, c->d4c, 4 * C, false, W(c, pi(FC_W)), C, true, e));
    }
    {
      PROF(PROF_LN_BWD, 0, ln_bwd_bytes);
      // the new dres is d loss / d x1: its column sums are this layer's attn.c_proj bias gradient
      float* part = c->ln_part + (2 * l + 1) * ln_slot;
      RC(launch_layernorm_bwd(st, c->bf16, c->dy, a.x1, a.ln2_mean, a.ln2_rstd, P(c, pi(LN2_W)), c->dres,
                              c->dres_act, true, part, c->ln_blocks, N, C));
      ln_jobs(part, G(c, pi(LN2_W)), G(c, pi(LN2_B)), G(c, pi(PROJ_B)));
    }
    // ---- attention: x1 = x + attn(ln1 Wqkv^T + bqkv) Wp^T + bp
    e = epi_make(EPI_ACCUM_F32, G(c, pi(PROJ_W)), C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * Cd * Cd, 0);
      RC(gemm(c, C, C, N, c->dres_act, C, true, a.attn, C, true, e));
    }
    e = epi_make(EPI_STORE_ACT, c->dattn, C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * Cd * Cd, 0);
      RC(gemm(c, N, C, C, c->dres_act, C, false, W(c, pi(PROJ_W)), C, true, e));
    }
    // the tensor-core path also leaves the column sums of dqkv (the c_attn bias gradient) per
    // 32-row group, so dqkv is not read again for them
    const bool fused_qkv_bias = c->attn_bias_part != nullptr;
    float* qkv_part = fused_qkv_bias ? c->attn_bias_part + l * c->attn_bias_stride : nullptr;
    {
      PROF(PROF_ATTN_BWD, 4.0 * B * (double)T * T * Cd, 0);
      RC(launch_attn_bwd(st, c->bf16, a.qkv, a.attn, c->dattn, a.attn_lse, c->attnD, c->dqkv, B, T, H, hd,
                         qkv_part));
    }
    e = epi_make(EPI_ACCUM_F32, G(c, pi(ATTN_W)), C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * 3 * Cd * Cd, 0);
      RC(gemm(c, 3 * C, C, N, c->dqkv, 3 * C, true, a.ln1, C, true, e));
    }
    if (fused_qkv_bias) {
      jobs.push_back(ColsumJob{qkv_part, G(c, pi(ATTN_B)), 3 * C, attn_bwd_bias_rows(B, T), 3 * C});
    } else {
      PROF(PROF_BIAS, 0, A * Nd * 3 * Cd);
      RC(launch_colsum(st, c->bf16, c->dqkv, 3 * C, N, 3 * C, c->colsum_part, ncs, G(c, pi(ATTN_B))));
    }
    e = epi_make(dy_kind, c->dy, C);
    {
      PROF(PROF_GEMM_BWD, 2.0 * Nd * 3 * Cd * Cd, 0);
      RC(gemm(c, N, C, 3 * C, c->dqkv, 3 * C, false, W(c, pi(ATTN_W)), C, true, e));
    }
    {
      PROF(PROF_LN_BWD, 0, ln_bwd_bytes);
      // the new dres is d loss / d x_l: the previous layer's mlp.c_proj bias gradient
      float* db_prev = (l > 0) ? G(c, param_index(g, l - 1, MPROJ_B)) : nullptr;
      float* part = c->ln_part + 2 * l * ln_slot;
      RC(launch_layernorm_bwd(st, c->bf16, c->dy, x, a.ln1_mean, a.ln1_rstd, P(c, pi(LN1_W)), c->dres, c->dres_act,
                              true, part, c->ln_blocks, N, C));
      ln_jobs(part, G(c, pi(LN1_W)), G(c, pi(LN1_B)), db_prev);
    }
  }
  {
    double bytes = 0;
    for (const ColsumJob& j : jobs) bytes += 4.0 * j.rows * j.ncols;
    PROF(PROF_BIAS, 0, bytes);
    RC(launch_colsum_batch(st, jobs.data(), (int)jobs.size()));
  }
  // token + position embedding
  {
    PROF(PROF_EMBED, 0, 8.0 * Nd * Cd + 8.0 * T * Cd);
    RC(launch_encoder_bwd(st, c->tokens, c->dres, G(c, 0), G(c, 1), B, T, C, c->enc_sorted, c->enc_seg, c->enc_part,
                          g.vocab_size));
  }
  return GPT2_OK;
}

int validate_cfg(const gpt2_config* g) {
  if (g->n_layer <= 0 || g->n_embd <= 0 || g->n_head <= 0 || g->block_size <= 0 || g->vocab_size <= 0 ||
      g->max_batch <= 0 || g->grad_accum_steps <= 0)
    return GPT2_ERR_ARG;
  if (g->padded_vocab_size < g->vocab_size) return GPT2_ERR_ARG;
  if (g->precision != GPT2_FP32 && g->precision != GPT2_BF16) return GPT2_ERR_ARG;
  if (g->n_embd % g->n_head) return GPT2_ERR_SHAPE;
  const int hd = g->n_embd / g->n_head;
  if (hd != 16 && hd != 32 && hd != 64) return GPT2_ERR_SHAPE;
  if (g->n_embd % 32 || g->n_embd > 1024) return GPT2_ERR_SHAPE;
  if ((long long)g->max_batch * g->block_size > ENC_MAX_POSITIONS) return GPT2_ERR_SHAPE;
  if (g->padded_vocab_size >= 131072) return GPT2_ERR_SHAPE;
  return GPT2_OK;
}

int init_params_impl(gpt2_ctx* c, uint64_t seed) {
  for (size_t t = 0; t < c->views.size(); ++t) {
    const ParamView& v = c->views[t];
    if (v.std < 0) {
      RC(launch_fill(c->stream, c->params + v.off, v.n, v.fill));
    } else {
      const uint64_t state = splitmix64_host(seed, (uint64_t)t);
      RC(launch_init_normal(c->stream, c->params + v.off, v.n, state, v.std));
    }
  }
  return GPT2_OK;
}

int refresh_shadow(gpt2_ctx* c) {
  if (!c->bf16) return GPT2_OK;
  return launch_cast_bf16(c->stream, c->params, c->shadow, c->nparams);
}

}  // namespace

// Runs the launch sequence `body` (forward_impl or backward_impl) on the context stream:
// eagerly on the first call with a key, captured into a CUDA graph on the second, replayed
// after that.  A capture that fails turns graphs off for the context and runs `body` eagerly.
// Profiling runs eagerly (its events are recorded per launch).
template <class F>
static int run_graphed(gpt2_ctx* c, int kind, int B, int T, F body) {
  if (!c->use_graphs || c->prof_on) return body();
  gpt2_ctx::GraphEntry* g = nullptr;
  for (auto& e : c->graphs)
    if (e.kind == kind && e.B == B && e.T == T) g = &e;
  if (g == nullptr) {
    c->graphs.push_back(gpt2_ctx::GraphEntry{kind, B, T, 0, nullptr, 0});
    g = &c->graphs.back();
  }
  if (g->exec == nullptr) {
    if (g->calls++ == 0) return body();   // modules loaded, kernel attributes set
    if (cudaStreamBeginCapture(c->stream, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
      cudaGetLastError();
      c->use_graphs = false;
      return body();
    }
    const long long n0 = kernel_launch_count();
    const int rc = body();
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(c->stream, &graph);
    const long long n = kernel_launch_count() - n0;
    note_kernel_launches((int)-n);   // nothing ran while capturing
    if (rc != 0 || e != cudaSuccess || graph == nullptr) {
      if (graph) cudaGraphDestroy(graph);
      cudaGetLastError();
      c->use_graphs = false;
      return rc ? rc : body();
    }
    e = cudaGraphInstantiate(&g->exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
      g->exec = nullptr;
      cudaGetLastError();
      c->use_graphs = false;
      return body();
    }
    g->launches = n;
  }
  cudaError_t e = cudaGraphLaunch(g->exec, c->stream);
  if (e != cudaSuccess) return cuda_fail(c, e, "graph launch");
  note_kernel_launches((int)g->launches);
  return GPT2_OK;
}

// ====================================================================== C ABI
extern "C" {

int gpt2_create(const gpt2_config* cfg, uint64_t seed, gpt2_ctx** out) {
  if (out == nullptr || cfg == nullptr) return GPT2_ERR_ARG;
  *out = nullptr;
  int rc = validate_cfg(cfg);
  if (rc) return rc;
  gpt2_ctx* c = new gpt2_ctx();
  c->cfg = *cfg;
  c->bf16 = cfg->precision == GPT2_BF16;
  c->act = c->bf16 ? 2 : 4;
  cudaError_t e = cudaGetDevice(&c->device);
  if (e != cudaSuccess) {
    delete c;
    return GPT2_ERR_CUDA;
  }
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (c->bf16) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, c->device);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, c->device);
    if (major != 10) {
      delete c;
      return GPT2_ERR_ARG;   // the tcgen05 path needs sm_100
    }
  }
  {
    const char* ge = getenv("GPT2_B200_GRAPHS");
    c->use_graphs = !(ge && ge[0] == '0');
  }
  if (cudaStreamCreateWithFlags(&c->own_stream, cudaStreamNonBlocking) != cudaSuccess) {
    delete c;
    return GPT2_ERR_CUDA;
  }
  c->stream = c->own_stream;
  build_views(c);

  const gpt2_config& g = c->cfg;
  const long long C = g.n_embd, L = g.n_layer, Vp = g.padded_vocab_size;
  const int H = g.n_head;
  c->Nmax = g.max_batch * g.block_size;
  const long long N = c->Nmax;
  c->ldl = (Vp + 7) / 8 * 8;
  const size_t A = c->act;
#define AL(expr)           \
  do {                     \
    rc = (expr);           \
    if (rc) goto fail_out; \
  } while (0)
  AL(dalloc(c, &c->params, c->nparams));
  AL(dalloc(c, &c->grads, c->nparams));
  AL(dalloc(c, &c->m, c->nparams));
  AL(dalloc(c, &c->v, c->nparams));
  if (c->bf16) AL(dalloc(c, &c->shadow, c->nparams));
  c->layers.resize(L);
  for (int l = 0; l < L; ++l) {
    LayerActs& a = c->layers[l];
    AL(dalloc_bytes(c, &a.ln1, N * C * A));
    AL(dalloc(c, &a.ln1_mean, N));
    AL(dalloc(c, &a.ln1_rstd, N));
    AL(dalloc_bytes(c, &a.qkv, N * 3 * C * A));
    AL(dalloc_bytes(c, &a.attn, N * C * A));
    AL(dalloc(c, &a.attn_lse, N * H));
    AL(dalloc(c, &a.x1, N * C));
    AL(dalloc_bytes(c, &a.ln2, N * C * A));
    AL(dalloc(c, &a.ln2_mean, N));
    AL(dalloc(c, &a.ln2_rstd, N));
    AL(dalloc_bytes(c, &a.fc_pre, N * 4 * C * A));
    AL(dalloc_bytes(c, &a.fc_act, N * 4 * C * A));
  }
  AL(dalloc(c, &c->resid, (L + 1) * N * C));
  AL(dalloc_bytes(c, &c->lnf, N * C * A));
  AL(dalloc(c, &c->lnf_mean, N));
  AL(dalloc(c, &c->lnf_rstd, N));
  AL(dalloc_bytes(c, &c->logits, N * c->ldl * A));
  AL(dalloc(c, &c->ce_part, N * (size_t)gemm_tc_ce_tiles((int)Vp)));
  AL(dalloc(c, &c->zt, N));
  AL(dalloc(c, &c->lse, N));
  AL(dalloc(c, &c->loss_row, N));
  AL(dalloc(c, &c->argmax, N));
  AL(dalloc(c, &c->scalars, 8));
  AL(dalloc(c, &c->count, 4));
  AL(dalloc(c, &c->tokens, N));
  AL(dalloc(c, &c->targets, N));
  AL(dalloc(c, &c->dres, N * C));
  AL(dalloc_bytes(c, &c->dres_act, N * C * A));
  AL(dalloc_bytes(c, &c->dy, N * C * A));
  AL(dalloc_bytes(c, &c->d4c, N * 4 * C * A));
  AL(dalloc_bytes(c, &c->dqkv, N * 3 * C * A));
  AL(dalloc_bytes(c, &c->dattn, N * C * A));
  AL(dalloc(c, &c->attnD, N * H));
  if (c->bf16 && C / H == 64) {
    c->attn_bias_stride = (size_t)attn_bwd_bias_rows(g.max_batch, g.block_size) * 3 * C;
    AL(dalloc(c, &c->attn_bias_part, L * c->attn_bias_stride));
  }
  if (c->bf16) {
    c->fc_bias_stride = (size_t)cdiv(g.max_batch * g.block_size, 32) * 4 * C;
    AL(dalloc(c, &c->fc_bias_part, L * c->fc_bias_stride));
  }
  c->ln_blocks = layernorm_bwd_blocks(c->num_sms);
  AL(dalloc(c, &c->ln_part, (2 * L + 1) * (size_t)c->ln_blocks * 3 * C));
  AL(dalloc(c, &c->colsum_part, (size_t)colsum_chunks((int)N) * 4 * C));
  AL(dalloc(c, &c->enc_sorted, N));
  AL(dalloc(c, &c->enc_seg, encoder_bwd_seg_words((int)N)));
  AL(dalloc(c, &c->enc_part, encoder_bwd_part_floats((int)N, (int)C)));
  c->splitk_ws_elems = (size_t)8 * 4 * C * C;
  AL(dalloc(c, &c->splitk_ws, c->splitk_ws_elems));
  c->norm_nparts = 4 * c->num_sms;
  AL(dalloc(c, &c->norm_part, c->norm_nparts));
  {
    // AdamW block table: each tensor split into blocks of 8192 elements; the kernel's 16-byte
    // accesses need every block to start and end on a multiple of 4 elements
    std::vector<AdamBlock> blocks;
    for (const ParamView& v : c->views) {
      if (v.off % 4 || v.n % 4) {
        rc = GPT2_ERR_SHAPE;
        goto fail_out;
      }
      for (long long o = 0; o < v.n; o += 8192) {
        AdamBlock b;
        b.off = v.off + o;
        b.n = (int)std::min<long long>(8192, v.n - o);
        b.decay = v.decay;
        blocks.push_back(b);
      }
    }
    c->n_adam_blocks = (int)blocks.size();
    AL(dalloc(c, &c->adam_blocks, blocks.size()));
    if (h2d_ordered(c, c->adam_blocks, blocks.data(), blocks.size() * sizeof(AdamBlock)) !=
        cudaSuccess) {
      rc = GPT2_ERR_CUDA;
      goto fail_out;
    }
  }
  if (cudaMemsetAsync(c->grads, 0, c->nparams * sizeof(float), c->stream) != cudaSuccess ||
      cudaMemsetAsync(c->m, 0, c->nparams * sizeof(float), c->stream) != cudaSuccess ||
      cudaMemsetAsync(c->v, 0, c->nparams * sizeof(float), c->stream) != cudaSuccess) {
    rc = GPT2_ERR_CUDA;
    goto fail_out;
  }
  AL(init_params_impl(c, seed));
  AL(refresh_shadow(c));
  rc = check_device(c);
  if (rc) goto fail_out;
#undef AL
  *out = c;
  return GPT2_OK;
fail_out:
  gpt2_destroy(c);
  return rc;
}

void gpt2_destroy(gpt2_ctx* c) {
  if (c == nullptr) return;
  if (c->stream) cudaStreamSynchronize(c->stream);
  for (auto& g : c->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  for (cudaEvent_t e : c->prof_events) cudaEventDestroy(e);
  for (void* p : c->allocs) cudaFree(p);
  if (c->own_stream) cudaStreamDestroy(c->own_stream);
  delete c;
}

int gpt2_set_stream(gpt2_ctx* c, void* s) {
  if (c == nullptr) return GPT2_ERR_ARG;
  c->stream = s ? reinterpret_cast<cudaStream_t>(s) : c->own_stream;
  return GPT2_OK;
}

int gpt2_set_graphs(gpt2_ctx* c, int enable) {
  if (c == nullptr) return GPT2_ERR_ARG;
  c->use_graphs = enable != 0;
  return GPT2_OK;
}

static int forward_common(gpt2_ctx* c, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out,
                          cudaMemcpyKind kind) {
  if (c == nullptr || tokens == nullptr) return fail(c, GPT2_ERR_ARG, "null argument");
  if (B <= 0 || T <= 0 || B > c->cfg.max_batch || T > c->cfg.block_size)
    return fail(c, GPT2_ERR_SHAPE, "B or T outside [1, max_batch] x [1, block_size]");
  const size_t bytes = (size_t)B * T * sizeof(int32_t);
  cudaError_t e = cudaMemcpyAsync(c->tokens, tokens, bytes, kind, c->stream);
  if (e != cudaSuccess) return cuda_fail(c, e, "token copy");
  if (targets) {
    e = cudaMemcpyAsync(c->targets, targets, bytes, kind, c->stream);
    if (e != cudaSuccess) return cuda_fail(c, e, "target copy");
  }
  c->lastB = B;
  c->lastT = T;
  c->have_targets = false;
  c->have_logits = false;
  const bool with_t = targets != nullptr;
  int rc = run_graphed(c, with_t ? 1 : 0, B, T, [&] { return forward_impl(c, B, T, with_t); });
  if (rc) return rc;
  c->have_targets = with_t;
  c->have_logits = true;
  if (loss_out) {
    rc = check_device(c);
    if (rc) return rc;
    if (!targets) return fail(c, GPT2_ERR_ARG, "loss requested without targets");
    e = cudaMemcpy(loss_out, &c->scalars[0], sizeof(float), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(c, e, "loss read");
  }
  return GPT2_OK;
}

int gpt2_forward(gpt2_ctx* c, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out) {
  return forward_common(c, tokens, targets, B, T, loss_out, cudaMemcpyDeviceToDevice);
}

int gpt2_forward_host(gpt2_ctx* c, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out) {
  return forward_common(c, tokens, targets, B, T, loss_out, cudaMemcpyHostToDevice);
}

int gpt2_backward(gpt2_ctx* c) {
  if (c == nullptr) return GPT2_ERR_ARG;
  if (!c->have_targets) return fail(c, GPT2_ERR_STATE, "backward needs a preceding forward with targets");
  int rc = run_graphed(c, 2, c->lastB, c->lastT, [&] { return backward_impl(c); });
  c->have_targets = false;   // the logits buffer now holds their gradient
  c->have_logits = false;
  return rc;
}

int gpt2_sample_top_k(gpt2_ctx* c, const int32_t* rows, const float* u, int n, int k, int32_t* out,
                      int32_t* out_topk) {
  if (c == nullptr || rows == nullptr || u == nullptr || out == nullptr) return fail(c, GPT2_ERR_ARG, "null argument");
  if (!c->have_logits) return fail(c, GPT2_ERR_STATE, "sampling needs the logits of a forward with no backward since");
  if (n <= 0 || k <= 0 || k > GPT2_SAMPLE_MAX_K) return fail(c, GPT2_ERR_SHAPE, "n <= 0 or k outside [1, 1024]");
  const int rc = launch_topk_sample(c->stream, c->bf16, c->logits, c->ldl, c->lastB * c->lastT, rows, u, n,
                                    c->cfg.vocab_size, k, out, out_topk);
  if (rc == -4) return fail(c, GPT2_ERR_SHAPE, "sampling shape");
  return rc ? fail(c, GPT2_ERR_CUDA, "sampling launch") : GPT2_OK;
}

int gpt2_get_grad_buffer(gpt2_ctx* c, float** device_ptr, int64_t* n) {
  if (c == nullptr || device_ptr == nullptr || n == nullptr) return GPT2_ERR_ARG;
  *device_ptr = c->grads;
  *n = (int64_t)c->nparams;
  return GPT2_OK;
}

int gpt2_zero_grad(gpt2_ctx* c) {
  if (c == nullptr) return GPT2_ERR_ARG;
  cudaError_t e = cudaMemsetAsync(c->grads, 0, c->nparams * sizeof(float), c->stream);
  return e == cudaSuccess ? GPT2_OK : cuda_fail(c, e, "zero_grad");
}

int gpt2_adamw_step(gpt2_ctx* c, float lr, float beta1, float beta2, float eps, float wd, float clip,
                    float* grad_norm_out) {
  if (c == nullptr) return GPT2_ERR_ARG;
  if (!(clip > 0.f) || !(eps >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
    return fail(c, GPT2_ERR_ARG, "invalid optimizer hyper-parameter");
  {
    PROF(PROF_OPTIM, 0, 4.0 * c->nparams);
    RC(launch_global_norm(c->stream, c->grads, c->nparams, c->norm_part, c->norm_nparts, clip, &c->scalars[2]));
  }
  c->step_t += 1;
  const double bc1 = 1.0 - std::pow((double)beta1, (double)c->step_t);
  const double bc2 = 1.0 - std::pow((double)beta2, (double)c->step_t);
  {
    PROF(PROF_OPTIM, 0, 28.0 * c->nparams + (c->bf16 ? 2.0 * c->nparams : 0.0));
    RC(launch_adamw(c->stream, c->params, c->grads, c->m, c->v, c->bf16 ? c->shadow : nullptr, c->adam_blocks,
                    c->n_adam_blocks, &c->scalars[3], lr, beta1, beta2, eps, wd, (float)bc1, (float)bc2));
  }
  if (grad_norm_out) {
    int rc = check_device(c);
    if (rc) return rc;
    cudaError_t e = cudaMemcpy(grad_norm_out, &c->scalars[2], sizeof(float), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(c, e, "norm read");
  }
  return GPT2_OK;
}

int64_t gpt2_num_params(const gpt2_ctx* c) { return c ? c->nparams : 0; }

static int copy_out(gpt2_ctx* c, void* dst, const void* src, size_t bytes) {
  if (c == nullptr || dst == nullptr) return GPT2_ERR_ARG;
  int rc = check_device(c);
  if (rc) return rc;
  cudaError_t e = cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? GPT2_OK : cuda_fail(c, e, "device to host copy");
}

int gpt2_get_params(gpt2_ctx* c, float* dst) {
  return copy_out(c, dst, c ? c->params : nullptr, c ? c->nparams * sizeof(float) : 0);
}
int gpt2_get_grads(gpt2_ctx* c, float* dst) {
  return copy_out(c, dst, c ? c->grads : nullptr, c ? c->nparams * sizeof(float) : 0);
}
int gpt2_set_params(gpt2_ctx* c, const float* src) {
  if (c == nullptr || src == nullptr) return GPT2_ERR_ARG;
  int rc = check_device(c);
  if (rc) return rc;
  cudaError_t e = h2d_ordered(c, c->params, src, c->nparams * sizeof(float));
  if (e != cudaSuccess) return cuda_fail(c, e, "set_params copy");
  RC(refresh_shadow(c));
  return check_device(c);
}
int gpt2_get_optimizer_state(gpt2_ctx* c, float* m_dst, float* v_dst, int64_t* t_out) {
  if (c == nullptr) return GPT2_ERR_ARG;
  if (m_dst) RC(copy_out(c, m_dst, c->m, c->nparams * sizeof(float)));
  if (v_dst) RC(copy_out(c, v_dst, c->v, c->nparams * sizeof(float)));
  if (t_out) *t_out = c->step_t;
  return GPT2_OK;
}
int gpt2_set_optimizer_state(gpt2_ctx* c, const float* m_src, const float* v_src, int64_t t) {
  if (c == nullptr || m_src == nullptr || v_src == nullptr || t < 0) return GPT2_ERR_ARG;
  int rc = check_device(c);
  if (rc) return rc;
  if (h2d_ordered(c, c->m, m_src, c->nparams * sizeof(float)) != cudaSuccess ||
      h2d_ordered(c, c->v, v_src, c->nparams * sizeof(float)) != cudaSuccess)
    return fail(c, GPT2_ERR_CUDA, "set_optimizer_state copy");
  c->step_t = t;
  return GPT2_OK;
}
int gpt2_get_argmax(gpt2_ctx* c, int32_t* dst) {
  return copy_out(c, dst, c ? c->argmax : nullptr, c ? (size_t)c->lastB * c->lastT * sizeof(int) : 0);
}
int gpt2_get_lse(gpt2_ctx* c, float* dst) {
  return copy_out(c, dst, c ? c->lse : nullptr, c ? (size_t)c->lastB * c->lastT * sizeof(float) : 0);
}
int gpt2_get_loss(gpt2_ctx* c, float* loss_out) {
  return copy_out(c, loss_out, c ? &c->scalars[0] : nullptr, sizeof(float));
}
int gpt2_synchronize(gpt2_ctx* c) {
  if (c == nullptr) return GPT2_ERR_ARG;
  return check_device(c);
}
const char* gpt2_last_error(const gpt2_ctx* c) { return c ? c->err.c_str() : "null context"; }

double gpt2_lr_cosine(int64_t it, double max_lr, int64_t warmup_steps, int64_t max_steps, double min_ratio) {
  const double min_lr = max_lr * min_ratio;
  if (it < warmup_steps) return max_lr * (double)(it + 1) / (double)warmup_steps;
  if (it > max_steps) return min_lr;
  const double r = (double)(it - warmup_steps) / (double)(max_steps - warmup_steps);
  return min_lr + 0.5 * (1.0 + std::cos(M_PI * r)) * (max_lr - min_lr);
}

int64_t gpt2_kernel_launches(void) { return kernel_launch_count(); }

int gpt2_profile_start(gpt2_ctx* c) {
  if (c == nullptr) return GPT2_ERR_ARG;
  c->prof_on = true;
  c->prof_used = 0;
  c->prof_class.clear();
  for (int i = 0; i < GPT2_PROF_CLASSES; ++i) {
    c->prof_flops[i] = 0;
    c->prof_bytes[i] = 0;
    c->prof_launches[i] = 0;
  }
  return GPT2_OK;
}

int gpt2_profile_stop(gpt2_ctx* c, double* ms, int64_t* launches, double* flops, double* bytes) {
  if (c == nullptr) return GPT2_ERR_ARG;
  c->prof_on = false;
  int rc = check_device(c);
  if (rc) return rc;
  double tot[GPT2_PROF_CLASSES] = {0};
  for (size_t i = 0; i < c->prof_class.size(); ++i) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, c->prof_events[2 * i], c->prof_events[2 * i + 1]) != cudaSuccess)
      return fail(c, GPT2_ERR_CUDA, "event timing failed");
    tot[c->prof_class[i]] += t;
  }
  for (int i = 0; i < GPT2_PROF_CLASSES; ++i) {
    if (ms) ms[i] = tot[i];
    if (launches) launches[i] = c->prof_launches[i];
    if (flops) flops[i] = c->prof_flops[i];
    if (bytes) bytes[i] = c->prof_bytes[i];
  }
  return GPT2_OK;
}

}  // extern "C"
