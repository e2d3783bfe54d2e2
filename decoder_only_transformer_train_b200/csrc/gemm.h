// GEMM interface shared by the tcgen05 (bf16) and SIMT (fp32 parity mode) kernels.
//
// Logical problem: D[m, n] = sum_k A(m, k) * B(n, k) for m < M, n < N, k < K, then an
// epilogue.  Each operand is either K-major (A(m,k) = A[m*lda + k]) or MN-major
// (A(m,k) = A[k*lda + m]), which covers the three products of a Linear layer
// y = x W^T + b:  forward  Y = X W^T        (A=X K-major,  B=W K-major)
//                 dX = dY W                 (A=dY K-major, B=W MN-major)
//                 dW += dY^T X              (A=dY MN-major, B=X MN-major)
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

enum EpiKind : int {
  EPI_STORE_ACT = 0,   // C(act) = alpha*D + bias
  EPI_STORE_F32 = 1,   // C(f32) = alpha*D + bias
  EPI_ACCUM_F32 = 2,   // C(f32) += alpha*D                 (weight gradients)
  EPI_RESID_F32 = 3,   // C(f32) = aux(f32) + alpha*D + bias (residual stream)
  EPI_GELU_FWD = 4,    // u = alpha*D + bias; aux_out(act) = gelu'(u); C(act) = gelu(u)
  EPI_GELU_BWD = 5,    // C(act) = alpha*D * aux(act)   (aux: the gelu'(u) the forward kept); optional
                       // column sums of C per 32-row group (the c_fc bias gradient's partials)
  EPI_CE_FWD = 6,      // C(act) = alpha*D (logits) + per-(row, column-tile) softmax partials
  EPI_SPLITK = 7,      // ws[split][m][n] = D   (internal: split-K partial products)
};

struct CePartial {      // per (row, column tile) of the logits
  float max;            // max logit of the tile
  float sum;            // sum of exp(logit - max) over the tile
  float amax;           // max logit value (same as max, kept for clarity of the argmax)
  int aidx;             // lowest column index reaching amax
};

struct EpiParams {
  int kind;
  int M, N;
  void* C;
  long long ldc;
  const float* bias;
  float alpha;
  const void* aux;
  long long ld_aux;
  void* aux_out;
  long long ld_aux_out;
  // EPI_CE_FWD
  const int* targets;   // [M]; -1 = ignored
  CePartial* ce_part;   // [M][n_ctiles]
  float* zt;            // [M] logit of the target column
  int n_ctiles;         // number of column tiles of the launch (set by the launcher)
  int ce_tile_n;        // column-tile width of the partials (set by the launcher)
  // EPI_SPLITK
  float* ws;
  int kb_per_split;
  // EPI_GELU_BWD (optional): column sums of C before its bf16 rounding, one fp32 row per
  // 32-row group: colsum_part[(m / 32) * N + n] = sum over the group's rows m < M of C[m, n]
  float* colsum_part;
};

inline EpiParams epi_make(int kind, void* C, long long ldc) {
  EpiParams e{};
  e.kind = kind;
  e.C = C;
  e.ldc = ldc;
  e.alpha = 1.0f;
  return e;
}

// bf16 tcgen05 GEMM.  `ws` (may be null) is fp32 workspace for split-K of EPI_ACCUM_F32
// problems with few output tiles and a long K; ws_elems is its size in floats.
// Returns 0 or a negative error code.
int gemm_bf16_tc(cudaStream_t st, int M, int N, int K, const void* A, long long lda, bool a_mn,
                 const void* B, long long ldb, bool b_mn, EpiParams ep, float* ws, size_t ws_elems,
                 int num_sms);

// fp32 SIMT GEMM (parity mode).  act type is float.
int gemm_f32_simt(cudaStream_t st, int M, int N, int K, const float* A, long long lda, bool a_mn,
                  const float* B, long long ldb, bool b_mn, EpiParams ep);

// Output tile width of the tcgen05 GEMM for a given N.
int gemm_tc_tile_n(int N);
// Number of per-row softmax partials EPI_CE_FWD writes for N columns (two per tile).
int gemm_tc_ce_tiles(int N);
