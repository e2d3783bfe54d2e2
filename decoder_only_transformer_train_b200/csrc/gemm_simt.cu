// fp32 SIMT GEMM used by the fp32 parity mode of the library (true fp32 products: the
// tensor-core TF32 path is not accurate enough for the 1e-4 fp32 parity bar).  Same
// operand conventions and epilogue semantics as the tcgen05 kernel, element by element.
#include "common.cuh"
#include "gemm.h"
#include "kernels.h"

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__device__ __forceinline__ void epi_elem_f32(const EpiParams& ep, int m, int n, float v) {
  const float b = (ep.bias != nullptr) ? ep.bias[n] : 0.0f;
  float* C = reinterpret_cast<float*>(ep.C) + (long long)m * ep.ldc + n;
  switch (ep.kind) {
    case EPI_STORE_ACT:
    case EPI_STORE_F32:
      *C = ep.alpha * v + b;
      break;
    case EPI_ACCUM_F32:
      *C += ep.alpha * v;
      break;
    case EPI_RESID_F32:
      *C = reinterpret_cast<const float*>(ep.aux)[(long long)m * ep.ld_aux + n] + ep.alpha * v + b;
      break;
    case EPI_GELU_FWD: {
      float g, gp;
      gelu_tanh_and_grad_f(ep.alpha * v + b, g, gp);
      reinterpret_cast<float*>(ep.aux_out)[(long long)m * ep.ld_aux_out + n] = gp;
      *C = g;
      break;
    }
    case EPI_GELU_BWD:
      *C = ep.alpha * v * reinterpret_cast<const float*>(ep.aux)[(long long)m * ep.ld_aux + n];
      break;
    default:
      break;
  }
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(256) gemm_simt_kernel(int M, int N, int K, const float* __restrict__ A,
                                                        long long lda, const float* __restrict__ B, long long ldb,
                                                        EpiParams ep) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      int mm, kk;
      if (A_MN) { mm = i % TM; kk = i / TM; } else { kk = i % TK; mm = i / TK; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? (A_MN ? A[(long long)gk * lda + gm] : A[(long long)gm * lda + gk]) : 0.0f;
    }
    for (int i = threadIdx.x; i < TN * TK; i += 256) {
      int nn, kk;
      if (B_MN) { nn = i % TN; kk = i / TN; } else { kk = i % TK; nn = i / TK; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < N && gk < K) ? (B_MN ? B[(long long)gk * ldb + gn] : B[(long long)gn * ldb + gk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) epi_elem_f32(ep, m, n, acc[i][j]);
    }
}

}  // namespace

int gemm_f32_simt(cudaStream_t st, int M, int N, int K, const float* A, long long lda, bool a_mn, const float* B,
                  long long ldb, bool b_mn, EpiParams ep) {
  if (M <= 0 || N <= 0) return 0;
  if (ep.kind == EPI_CE_FWD || ep.kind == EPI_SPLITK) return -1;
  ep.M = M;
  ep.N = N;
  dim3 grid(cdiv(N, TN), cdiv(M, TM));
  if (!a_mn && !b_mn) gemm_simt_kernel<false, false><<<grid, 256, 0, st>>>(M, N, K, A, lda, B, ldb, ep);
  else if (!a_mn && b_mn) gemm_simt_kernel<false, true><<<grid, 256, 0, st>>>(M, N, K, A, lda, B, ldb, ep);
  else if (a_mn && b_mn) gemm_simt_kernel<true, true><<<grid, 256, 0, st>>>(M, N, K, A, lda, B, ldb, ep);
  else gemm_simt_kernel<true, false><<<grid, 256, 0, st>>>(M, N, K, A, lda, B, ldb, ep);
  note_kernel_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
