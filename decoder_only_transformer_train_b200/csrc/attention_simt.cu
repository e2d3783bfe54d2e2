// Causal self-attention, forward and backward, as flash attention: keys and values are
// streamed through shared memory in 64-row tiles with an online softmax (running max and
// sum, Milakov & Gimelshein 2018), so the T x T score matrix is never stored; the
// backward recomputes the probabilities from the saved log-sum-exp.  ("Karpathy's Zero to
// Hero, Lecture 9" notes, "2:00:19 – 2:06:39 FlashAttention".)
//
// This SIMT version (fp32 arithmetic, one thread per query or key row) serves the fp32
// parity mode and any head size up to 64.
//
// Layout: qkv [B*T, 3C] with q | k | v column blocks and head h at columns h*hd .. +hd;
// out [B*T, C] (heads re-assembled); lse [B, H, T]; scale 1/sqrt(hd).
#include <math.h>
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int AT = 64;   // rows per tile

// Same for bf16 with head size 64: a warp per token row (all heads), 16-byte loads; lane l
// takes the 8-channel groups l, l + 32, ... and the 8 lanes of a head add by shuffles.
__global__ void __launch_bounds__(256) attn_bwd_D_bf16_hd64(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                                            float* __restrict__ Dbuf, int Tn, int H, long long ntok) {
  const long long tok = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= ntok) return;                     // warp-uniform
  const int groups = H * 8;                    // 8-channel groups per row
  const uint4* o = reinterpret_cast<const uint4*>(out) + tok * groups;
  const uint4* g = reinterpret_cast<const uint4*>(dout) + tok * groups;
  const long long b = tok / Tn;
  const int t = (int)(tok - b * Tn);
  for (int base = 0; base < groups; base += 32) {
    const int c8 = base + lane;
    float s = 0.f;
    if (c8 < groups) {
      const uint4 a = __ldcs(o + c8), d = __ldcs(g + c8);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 af = unpack_bf16x2(aw[i]), df = unpack_bf16x2(dw[i]);
        s = fmaf(af.x, df.x, s);
        s = fmaf(af.y, df.y, s);
      }
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (c8 < groups && (lane & 7) == 0) Dbuf[(b * H + (c8 >> 3)) * Tn + t] = s;
  }
}

template <typename T, int HD>
__global__ void __launch_bounds__(AT) attn_fwd_simt(const T* __restrict__ qkv, T* __restrict__ out,
                                                    float* __restrict__ lse, int Tn, int H, float scale) {
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD, ld = 3 * C;
  const int qb = blockIdx.x;
  const int i = qb * AT + threadIdx.x;
  __shared__ float Ks[AT][HD + 1], Vs[AT][HD + 1];
  const T* base = qkv + (long long)b * Tn * ld;
  float q[HD], o[HD];
  float m = -INFINITY, l = 0.f;
#pragma unroll
  for (int d = 0; d < HD; ++d) {
    q[d] = (i < Tn) ? ld_f(base + (long long)i * ld + h * HD + d) * scale : 0.f;
    o[d] = 0.f;
  }
  for (int kb = 0; kb <= qb; ++kb) {
    __syncthreads();
    for (int e = threadIdx.x; e < AT * HD; e += AT) {
      const int r = e / HD, d = e % HD, j = kb * AT + r;
      Ks[r][d] = (j < Tn) ? ld_f(base + (long long)j * ld + C + h * HD + d) : 0.f;
      Vs[r][d] = (j < Tn) ? ld_f(base + (long long)j * ld + 2 * C + h * HD + d) : 0.f;
    }
    __syncthreads();
    if (i < Tn) {
      const int jn = min(AT, i - kb * AT + 1);
      for (int jj = 0; jj < jn; ++jj) {
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < HD; ++d) s = fmaf(q[d], Ks[jj][d], s);
        if (s > m) {
          const float c = expf(m - s);
          l *= c;
#pragma unroll
          for (int d = 0; d < HD; ++d) o[d] *= c;
          m = s;
        }
        const float p = expf(s - m);
        l += p;
#pragma unroll
        for (int d = 0; d < HD; ++d) o[d] = fmaf(p, Vs[jj][d], o[d]);
      }
    }
  }
  if (i < Tn) {
    const float inv = 1.0f / l;
    T* orow = out + ((long long)b * Tn + i) * C + h * HD;
#pragma unroll
    for (int d = 0; d < HD; ++d) st_f(orow + d, o[d] * inv);
    lse[(long long)bh * Tn + i] = m + logf(l);
  }
}

// D[b,h,i] = sum_d dO[i,d] * O[i,d]   (= rowsum(dP * P) of the softmax backward)
template <typename T>
__global__ void attn_bwd_D(const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ Dbuf, int Tn,
                           int H, int HD) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * 8LL + warp;   // over B*T*H rows (b, t, h)
  const int C = H * HD;
  const int b = blockIdx.y;
  if (row >= (long long)Tn * H) return;
  const int t = (int)(row / H), h = (int)(row % H);
  const long long off = ((long long)b * Tn + t) * C + h * HD;
  float s = 0.f;
  for (int d = lane; d < HD; d += 32) s += ld_f(dout + off + d) * ld_f(out + off + d);
  s = warp_sum(s);
  if (lane == 0) Dbuf[((long long)b * H + h) * Tn + t] = s;
}

template <typename T, int HD>
__global__ void __launch_bounds__(AT) attn_bwd_dkdv_simt(const T* __restrict__ qkv, const T* __restrict__ dout,
                                                         const float* __restrict__ lse, const float* __restrict__ Dbuf,
                                                         T* __restrict__ dqkv, int Tn, int H, float scale) {
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD, ld = 3 * C;
  const int kb = blockIdx.x;
  const int j = kb * AT + threadIdx.x;
  extern __shared__ float sm[];
  float(*Qs)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(sm);
  float(*dOs)[HD + 1] = Qs + AT;
  float(*Ko)[HD + 1] = dOs + AT;
  float(*Vo)[HD + 1] = Ko + AT;
  float* lse_s = reinterpret_cast<float*>(Vo + AT);
  float* D_s = lse_s + AT;
  const T* base = qkv + (long long)b * Tn * ld;
  for (int e = threadIdx.x; e < AT * HD; e += AT) {
    const int r = e / HD, d = e % HD, jj = kb * AT + r;
    Ko[r][d] = (jj < Tn) ? ld_f(base + (long long)jj * ld + C + h * HD + d) : 0.f;
    Vo[r][d] = (jj < Tn) ? ld_f(base + (long long)jj * ld + 2 * C + h * HD + d) : 0.f;
  }
  float dk[HD], dv[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) { dk[d] = 0.f; dv[d] = 0.f; }
  const int nqb = cdiv(Tn, AT);
  const T* dbase = dout + (long long)b * Tn * C;
  for (int qb = kb; qb < nqb; ++qb) {
    __syncthreads();
    for (int e = threadIdx.x; e < AT * HD; e += AT) {
      const int r = e / HD, d = e % HD, i = qb * AT + r;
      Qs[r][d] = (i < Tn) ? ld_f(base + (long long)i * ld + h * HD + d) : 0.f;
      dOs[r][d] = (i < Tn) ? ld_f(dbase + (long long)i * C + h * HD + d) : 0.f;
    }
    {
      const int i = qb * AT + threadIdx.x;
      lse_s[threadIdx.x] = (i < Tn) ? lse[(long long)bh * Tn + i] : 0.f;
      D_s[threadIdx.x] = (i < Tn) ? Dbuf[(long long)bh * Tn + i] : 0.f;
    }
    __syncthreads();
    if (j < Tn) {
      for (int ii = 0; ii < AT; ++ii) {
        const int i = qb * AT + ii;
        if (i >= Tn) break;
        if (i < j) continue;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
          s = fmaf(Qs[ii][d], Ko[threadIdx.x][d], s);
          dp = fmaf(dOs[ii][d], Vo[threadIdx.x][d], dp);
        }
        const float p = expf(s * scale - lse_s[ii]);
        const float ds = p * (dp - D_s[ii]) * scale;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
          dv[d] = fmaf(p, dOs[ii][d], dv[d]);
          dk[d] = fmaf(ds, Qs[ii][d], dk[d]);
        }
      }
    }
  }
  if (j < Tn) {
    T* row = dqkv + ((long long)b * Tn + j) * ld + h * HD;
#pragma unroll
    for (int d = 0; d < HD; ++d) {
      st_f(row + C + d, dk[d]);
      st_f(row + 2 * C + d, dv[d]);
    }
  }
}

template <typename T, int HD>
__global__ void __launch_bounds__(AT) attn_bwd_dq_simt(const T* __restrict__ qkv, const T* __restrict__ dout,
                                                       const float* __restrict__ lse, const float* __restrict__ Dbuf,
                                                       T* __restrict__ dqkv, int Tn, int H, float scale) {
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int C = H * HD, ld = 3 * C;
  const int qb = blockIdx.x;
  const int i = qb * AT + threadIdx.x;
  extern __shared__ float sm[];
  float(*Ks)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(sm);
  float(*Vs)[HD + 1] = Ks + AT;
  float(*dOo)[HD + 1] = Vs + AT;
  const T* base = qkv + (long long)b * Tn * ld;
  float q[HD], dq[HD];
#pragma unroll
  for (int d = 0; d < HD; ++d) {
    q[d] = (i < Tn) ? ld_f(base + (long long)i * ld + h * HD + d) : 0.f;
    dq[d] = 0.f;
  }
  const T* dbase = dout + (long long)b * Tn * C;
  for (int e = threadIdx.x; e < AT * HD; e += AT) {
    const int r = e / HD, d = e % HD, ii = qb * AT + r;
    dOo[r][d] = (ii < Tn) ? ld_f(dbase + (long long)ii * C + h * HD + d) : 0.f;
  }
  const float li = (i < Tn) ? lse[(long long)bh * Tn + i] : 0.f;
  const float Di = (i < Tn) ? Dbuf[(long long)bh * Tn + i] : 0.f;
  for (int kb = 0; kb <= qb; ++kb) {
    __syncthreads();
    for (int e = threadIdx.x; e < AT * HD; e += AT) {
      const int r = e / HD, d = e % HD, j = kb * AT + r;
      Ks[r][d] = (j < Tn) ? ld_f(base + (long long)j * ld + C + h * HD + d) : 0.f;
      Vs[r][d] = (j < Tn) ? ld_f(base + (long long)j * ld + 2 * C + h * HD + d) : 0.f;
    }
    __syncthreads();
    if (i < Tn) {
      const int jn = min(AT, i - kb * AT + 1);
      for (int jj = 0; jj < jn; ++jj) {
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
          s = fmaf(q[d], Ks[jj][d], s);
          dp = fmaf(dOo[threadIdx.x][d], Vs[jj][d], dp);
        }
        const float p = expf(s * scale - li);
        const float ds = p * (dp - Di) * scale;
#pragma unroll
        for (int d = 0; d < HD; ++d) dq[d] = fmaf(ds, Ks[jj][d], dq[d]);
      }
    }
  }
  if (i < Tn) {
    T* row = dqkv + ((long long)b * Tn + i) * ld + h * HD;
#pragma unroll
    for (int d = 0; d < HD; ++d) st_f(row + d, dq[d]);
  }
}

template <typename T, int HD>
int fwd_run(cudaStream_t st, const void* qkv, void* out, float* lse, int B, int Tn, int H) {
  dim3 grid(cdiv(Tn, AT), B * H);
  attn_fwd_simt<T, HD><<<grid, AT, 0, st>>>(reinterpret_cast<const T*>(qkv), reinterpret_cast<T*>(out), lse, Tn, H,
                                            1.0f / sqrtf((float)HD));
  note_kernel_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

template <typename T, int HD>
int bwd_run(cudaStream_t st, const void* qkv, const void* out, const void* dout, const float* lse, float* Dbuf,
            void* dqkv, int B, int Tn, int H) {
  const float scale = 1.0f / sqrtf((float)HD);
  dim3 gD(cdiv(Tn * H, 8), B);
  attn_bwd_D<T><<<gD, 256, 0, st>>>(reinterpret_cast<const T*>(out), reinterpret_cast<const T*>(dout), Dbuf, Tn, H,
                                    HD);
  dim3 grid(cdiv(Tn, AT), B * H);
  const int smem = (4 * AT * (HD + 1) + 2 * AT) * (int)sizeof(float);
  auto k1 = attn_bwd_dkdv_simt<T, HD>;
  if (smem > 48 * 1024 && cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) return -3;
  k1<<<grid, AT, smem, st>>>(reinterpret_cast<const T*>(qkv), reinterpret_cast<const T*>(dout), lse, Dbuf,
                             reinterpret_cast<T*>(dqkv), Tn, H, scale);
  const int smem2 = 3 * AT * (HD + 1) * (int)sizeof(float);
  auto k2 = attn_bwd_dq_simt<T, HD>;
  if (smem2 > 48 * 1024 && cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2)) return -3;
  k2<<<grid, AT, smem2, st>>>(reinterpret_cast<const T*>(qkv), reinterpret_cast<const T*>(dout), lse, Dbuf,
                              reinterpret_cast<T*>(dqkv), Tn, H, scale);
  note_kernel_launches(3);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace

int launch_attn_fwd_simt(cudaStream_t st, bool is_bf16, const void* qkv, void* out, float* lse, int B, int T, int H,
                         int hd) {
  switch (hd) {
    case 16: return is_bf16 ? fwd_run<bf16, 16>(st, qkv, out, lse, B, T, H) : fwd_run<float, 16>(st, qkv, out, lse, B, T, H);
    case 32: return is_bf16 ? fwd_run<bf16, 32>(st, qkv, out, lse, B, T, H) : fwd_run<float, 32>(st, qkv, out, lse, B, T, H);
    case 64: return is_bf16 ? fwd_run<bf16, 64>(st, qkv, out, lse, B, T, H) : fwd_run<float, 64>(st, qkv, out, lse, B, T, H);
    default: return -4;
  }
}

int launch_attn_bwd_simt(cudaStream_t st, bool is_bf16, const void* qkv, const void* out, const void* dout,
                         const float* lse, float* Dbuf, void* dqkv, int B, int T, int H, int hd) {
  switch (hd) {
#define AB(HD) case HD: return is_bf16 ? bwd_run<bf16, HD>(st, qkv, out, dout, lse, Dbuf, dqkv, B, T, H) \
                                       : bwd_run<float, HD>(st, qkv, out, dout, lse, Dbuf, dqkv, B, T, H);
    AB(16) AB(32) AB(64)
#undef AB
    default: return -4;
  }
}

int launch_attn_fwd(cudaStream_t st, bool is_bf16, const void* qkv, void* out, float* lse, int B, int T, int H,
                    int hd) {
  if (is_bf16 && hd == 64) return launch_attn_fwd_tc(st, qkv, out, lse, B, T, H, hd);
  return launch_attn_fwd_simt(st, is_bf16, qkv, out, lse, B, T, H, hd);
}
int launch_attn_bwd(cudaStream_t st, bool is_bf16, const void* qkv, const void* out, const void* dout,
                    const float* lse, float* Dbuf, void* dqkv, int B, int T, int H, int hd, float* bias_part) {
  if (is_bf16 && hd == 64) {
    const long long ntok = (long long)B * T;
    if ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(dout)) % 16 == 0) {
      attn_bwd_D_bf16_hd64<<<(unsigned)cdivll(ntok, 8), 256, 0, st>>>(reinterpret_cast<const bf16*>(out),
                                                                       reinterpret_cast<const bf16*>(dout), Dbuf, T, H,
                                                                       ntok);
    } else {
      dim3 gD(cdiv(T * H, 8), B);
      attn_bwd_D<bf16><<<gD, 256, 0, st>>>(reinterpret_cast<const bf16*>(out), reinterpret_cast<const bf16*>(dout),
                                           Dbuf, T, H, hd);
    }
    note_kernel_launches(1);
    if (cudaGetLastError() != cudaSuccess) return -3;
    return launch_attn_bwd_tc(st, qkv, dout, lse, Dbuf, dqkv, B, T, H, hd, bias_part);
  }
  if (bias_part != nullptr) return -4;   // the column sums come only with the tensor-core path
  return launch_attn_bwd_simt(st, is_bf16, qkv, out, dout, lse, Dbuf, dqkv, B, T, H, hd);
}
