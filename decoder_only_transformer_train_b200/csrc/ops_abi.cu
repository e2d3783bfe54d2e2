// Single-operation entry points of gpt2_b200.h on caller buffers (device pointers), so
// that each kernel can be checked against a reference on its own.
#include "gpt2_b200.h"
#include "common.cuh"
#include "gemm.h"
#include "kernels.h"

namespace {
int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}
}  // namespace

extern "C" {

int gpt2op_gemm_bf16(void* stream, int M, int N, int K, const void* A, int64_t lda, int a_mn_major, const void* B,
                     int64_t ldb, int b_mn_major, void* C, int64_t ldc, int epilogue, const float* bias, float alpha,
                     float* workspace, int64_t ws_floats) {
  if (A == nullptr || B == nullptr || C == nullptr) return GPT2_ERR_ARG;
  if (M < 0 || N < 0 || K <= 0) return GPT2_ERR_SHAPE;
  int kind;
  switch (epilogue) {
    case 0: kind = EPI_STORE_ACT; break;
    case 1: kind = EPI_STORE_F32; break;
    case 2: kind = EPI_ACCUM_F32; break;
    default: return GPT2_ERR_ARG;
  }
  if (reinterpret_cast<uintptr_t>(bias) % 16) return GPT2_ERR_ARG;   // 16-byte bias reads in the epilogue
  EpiParams e = epi_make(kind, C, ldc);
  e.bias = bias;
  e.alpha = alpha;
  int rc = gemm_bf16_tc(reinterpret_cast<cudaStream_t>(stream), M, N, K, A, lda, a_mn_major != 0, B, ldb,
                        b_mn_major != 0, e, workspace, workspace ? (size_t)ws_floats : 0, sm_count());
  return rc == 0 ? GPT2_OK : (rc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA);
}

int gpt2op_gemm_bf16_fused(void* stream, int M, int N, int K, const void* A, int64_t lda, int a_mn_major,
                           const void* B, int64_t ldb, int b_mn_major, void* C, int64_t ldc, int epilogue,
                           const float* bias, float alpha, const void* aux, int64_t ld_aux, void* aux_out,
                           int64_t ld_aux_out) {
  if (A == nullptr || B == nullptr || C == nullptr) return GPT2_ERR_ARG;
  if (M < 0 || N < 0 || K <= 0) return GPT2_ERR_SHAPE;
  int kind;
  switch (epilogue) {
    case 3: kind = EPI_RESID_F32; break;
    case 4: kind = EPI_GELU_FWD; break;
    case 5: kind = EPI_GELU_BWD; break;
    default: return GPT2_ERR_ARG;
  }
  if ((kind == EPI_RESID_F32 || kind == EPI_GELU_BWD) && aux == nullptr) return GPT2_ERR_ARG;
  if (kind == EPI_GELU_FWD && aux_out == nullptr) return GPT2_ERR_ARG;
  if ((aux && ld_aux % 8) || (aux_out && ld_aux_out % 8)) return GPT2_ERR_ARG;
  // the epilogue reads bias and aux and writes aux_out with 16-byte accesses
  if ((reinterpret_cast<uintptr_t>(bias) | reinterpret_cast<uintptr_t>(aux) | reinterpret_cast<uintptr_t>(aux_out)) %
      16)
    return GPT2_ERR_ARG;
  EpiParams e = epi_make(kind, C, ldc);
  e.bias = (kind == EPI_GELU_BWD) ? nullptr : bias;
  e.alpha = alpha;
  e.aux = aux;
  e.ld_aux = ld_aux;
  e.aux_out = aux_out;
  e.ld_aux_out = ld_aux_out;
  int rc = gemm_bf16_tc(reinterpret_cast<cudaStream_t>(stream), M, N, K, A, lda, a_mn_major != 0, B, ldb,
                        b_mn_major != 0, e, nullptr, 0, sm_count());
  return rc == 0 ? GPT2_OK : (rc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA);
}

int gpt2op_attention_fwd(void* stream, int precision, const void* qkv, void* out, float* lse, int B, int T, int H,
                         int head_dim) {
  if (!qkv || !out || !lse) return GPT2_ERR_ARG;
  int rc = launch_attn_fwd(reinterpret_cast<cudaStream_t>(stream), precision == GPT2_BF16, qkv, out, lse, B, T, H,
                           head_dim);
  return rc == 0 ? GPT2_OK : (rc == -4 ? GPT2_ERR_SHAPE : (rc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA));
}

int gpt2op_attention_bwd(void* stream, int precision, const void* qkv, const void* out, const void* dout,
                         const float* lse, float* Dbuf, void* dqkv, int B, int T, int H, int head_dim) {
  if (!qkv || !out || !dout || !lse || !Dbuf || !dqkv) return GPT2_ERR_ARG;
  int rc = launch_attn_bwd(reinterpret_cast<cudaStream_t>(stream), precision == GPT2_BF16, qkv, out, dout, lse, Dbuf,
                           dqkv, B, T, H, head_dim);
  return rc == 0 ? GPT2_OK : (rc == -4 ? GPT2_ERR_SHAPE : (rc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA));
}

int gpt2op_layernorm_fwd(void* stream, int precision, const float* x, const float* w, const float* b, void* y,
                         float* mean, float* rstd, int N, int C) {
  if (!x || !w || !b || !y || !mean || !rstd) return GPT2_ERR_ARG;
  int rc = launch_layernorm_fwd(reinterpret_cast<cudaStream_t>(stream), precision == GPT2_BF16, x, w, b, y, mean,
                                rstd, N, C);
  return rc == 0 ? GPT2_OK : (rc == -4 ? GPT2_ERR_SHAPE : GPT2_ERR_CUDA);
}

int gpt2op_embedding_fwd(void* stream, const int32_t* tokens, const float* wte, const float* wpe, float* x, int B,
                         int T, int C, int V) {
  if (!tokens || !wte || !wpe || !x) return GPT2_ERR_ARG;
  if (B <= 0 || T <= 0 || C <= 0 || V <= 0 || C % 4 || (long long)B * T > INT32_MAX) return GPT2_ERR_SHAPE;
  const int rc = launch_encoder_fwd(reinterpret_cast<cudaStream_t>(stream), tokens, wte, wpe, x, B * T, T, C, V);
  return rc == 0 ? GPT2_OK : (rc == -4 ? GPT2_ERR_SHAPE : (rc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA));
}

// workspace of the embedding backward: the sorted keys (N uint64), the segment keys and the
// chunk partials, each starting on a 256-byte boundary
static int64_t round256(int64_t b) { return (b + 255) / 256 * 256; }
static int64_t embedding_keys_bytes(int N) { return round256((int64_t)N * 8); }
static int64_t embedding_seg_bytes(int N) { return round256((int64_t)encoder_bwd_seg_words(N) * 4); }

int64_t gpt2op_embedding_bwd_ws_bytes(int N, int C) {
  if (N <= 0 || C <= 0) return 0;
  return embedding_keys_bytes(N) + embedding_seg_bytes(N) + (int64_t)encoder_bwd_part_floats(N, C) * 4;
}

int gpt2op_embedding_bwd(void* stream, const int32_t* tokens, const float* dx0, float* dwte, float* dwpe, int B,
                         int T, int C, int V, void* ws) {
  if (!tokens || !dx0 || !dwte || !dwpe || !ws) return GPT2_ERR_ARG;
  if (B <= 0 || T <= 0 || C <= 0 || V <= 0 || C % 4 || (long long)B * T > ENC_MAX_POSITIONS) return GPT2_ERR_SHAPE;
  char* w = static_cast<char*>(ws);
  const int N = B * T;
  const int rc = launch_encoder_bwd(reinterpret_cast<cudaStream_t>(stream), tokens, dx0, dwte, dwpe, B, T, C,
                                    reinterpret_cast<uint64_t*>(w),
                                    reinterpret_cast<uint32_t*>(w + embedding_keys_bytes(N)),
                                    reinterpret_cast<float*>(w + embedding_keys_bytes(N) + embedding_seg_bytes(N)), V);
  return rc == 0 ? GPT2_OK : (rc == -4 ? GPT2_ERR_SHAPE : (rc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA));
}

int gpt2op_sample_top_k(void* stream, int precision, const void* logits, int64_t ld, int n_rows,
                        const int32_t* rows, const float* u, int n, int V, int k, int32_t* out, int32_t* out_topk) {
  if (!logits || !rows || !u || !out) return GPT2_ERR_ARG;
  if (precision != GPT2_FP32 && precision != GPT2_BF16) return GPT2_ERR_ARG;
  if (n <= 0 || n_rows <= 0 || V <= 0 || k <= 0 || k > GPT2_SAMPLE_MAX_K || ld < V) return GPT2_ERR_SHAPE;
  const int rc = launch_topk_sample(reinterpret_cast<cudaStream_t>(stream), precision == GPT2_BF16, logits, ld,
                                    n_rows, rows, u, n, V, k, out, out_topk);
  return rc == 0 ? GPT2_OK : (rc == -4 ? GPT2_ERR_SHAPE : GPT2_ERR_CUDA);
}

int64_t gpt2op_classifier_aux_floats(int N, int V) {
  const int ntiles = gemm_tc_ce_tiles(V);
  // partials (4 floats each), zt, loss_row, and 8 scalars
  return (int64_t)N * ntiles * 4 + 2LL * N + 8;
}

int gpt2op_classifier_fwd_bwd(void* stream, const void* h, const void* W, const int32_t* targets, int N, int V, int C,
                              void* logits_ws, int64_t ldl, float* aux_ws, float* loss, float* lse, int32_t* argmax,
                              float* dh, float* dW) {
  if (!h || !W || !targets || !logits_ws || !aux_ws || !loss || !lse || !argmax || !dh || !dW) return GPT2_ERR_ARG;
  if (N <= 0 || V <= 0 || C <= 0 || ldl < V || ldl % 8 || C % 8) return GPT2_ERR_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int nsm = sm_count();
  const int ntiles = gemm_tc_ce_tiles(V);
  CePartial* part = reinterpret_cast<CePartial*>(aux_ws);
  float* zt = aux_ws + (size_t)N * ntiles * 4;
  float* loss_row = zt + N;
  float* scal = loss_row + N;   // [0] loss (unused copy) [1] dz scale
  int* count = reinterpret_cast<int*>(scal + 4);
  EpiParams e = epi_make(EPI_CE_FWD, logits_ws, ldl);
  e.targets = targets;
  e.ce_part = part;
  e.zt = zt;
  if (gemm_bf16_tc(st, N, V, C, h, C, false, W, C, false, e, nullptr, 0, nsm)) return GPT2_ERR_CUDA;
  if (launch_ce_finalize(st, part, ntiles, zt, targets, N, V, lse, loss_row, argmax)) return GPT2_ERR_CUDA;
  if (launch_loss_reduce(st, loss_row, targets, N, 1.0f, loss, &scal[1], count)) return GPT2_ERR_CUDA;
  if (launch_ce_dz(st, true, logits_ws, ldl, lse, targets, &scal[1], N, V)) return GPT2_ERR_CUDA;
  e = epi_make(EPI_STORE_F32, dh, C);
  if (gemm_bf16_tc(st, N, C, V, logits_ws, ldl, false, W, C, true, e, nullptr, 0, nsm)) return GPT2_ERR_CUDA;
  e = epi_make(EPI_ACCUM_F32, dW, C);
  if (gemm_bf16_tc(st, V, C, N, logits_ws, ldl, true, h, C, true, e, nullptr, 0, nsm)) return GPT2_ERR_CUDA;
  return GPT2_OK;
}

int gpt2op_device_error(void) {
  int code = 0;
  if (read_and_clear_device_error(&code)) return GPT2_ERR_CUDA;
  switch (code) {
    case DEVERR_NONE: return GPT2_OK;
    case DEVERR_TOKEN: return GPT2_ERR_TOKEN;
    case DEVERR_TARGET: return GPT2_ERR_TARGET;
    case DEVERR_TIMEOUT: return GPT2_ERR_TIMEOUT;
    case DEVERR_ROW: return GPT2_ERR_ARG;
    default: return GPT2_ERR_CUDA;
  }
}

}  // extern "C"
