// Memory-bound kernels of the GPT-2 training step: embedding gather and its
// deterministic backward, LayerNorm forward/backward, bias-gradient column sums, the
// cross-entropy finalisation and its logit gradient, the global gradient norm, AdamW and
// the parameter initialisation.  Rows are handled one warp each with coalesced (or
// 128-bit) accesses and warp-shuffle reductions; every cross-block reduction is done in
// a fixed order so that results are bitwise reproducible.
//
// Citations name "Karpathy's Zero to Hero, Lecture 9: Reproduce GPT-2 (124M)" notes (L9)
// and a section on that page.
#include <float.h>
#include "common.cuh"
#include "kernels.h"

__device__ int g_device_error = 0;

#include <atomic>
#include <map>
#include <mutex>
#include <utility>
static std::atomic<long long> g_kernel_launches{0};

int per_device_once(const void* key, const std::function<int()>& compute) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -3;
  std::lock_guard<std::mutex> lock(mu);
  const auto k = std::make_pair(key, dev);
  const auto it = cache.find(k);
  if (it != cache.end()) return it->second;
  const int v = compute();
  if (v >= 0) cache[k] = v;
  return v;
}

int current_device_sms() {
  static const int tag = 0;
  const int n = per_device_once(&tag, [] {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                     cudaSuccess || sms <= 0)
      return -3;
    return sms;
  });
  return n > 0 ? n : 148;
}

int set_dynamic_smem_once(const void* func, int bytes) {
  const int rc = per_device_once(func, [=] {
    return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess ? 1 : -3;
  });
  return rc < 0 ? -3 : 0;
}
void note_kernel_launches(int n) { g_kernel_launches.fetch_add(n, std::memory_order_relaxed); }
long long kernel_launch_count() { return g_kernel_launches.load(std::memory_order_relaxed); }

int read_and_clear_device_error(int* code) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -3;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return -3;
  *code = v;
  return 0;
}

namespace {

// ================================================================ encoder forward
// x[n, :] = wte[tok[n], :] + wpe[n mod T, :]   (L9, "Code you'll write": forward pass).
// Out-of-range ids are reported and embed as zeros.
// Thread x of a block copies channels 4x .. 4x+3 of four rows per pass, the rows of a
// block's passes strided by the grid, so that four wte and four wpe loads are in flight.
__global__ void __launch_bounds__(256) encoder_fwd_kernel(const int* __restrict__ tok,
                                                          const float4* __restrict__ wte,
                                                          const float4* __restrict__ wpe, float4* __restrict__ x,
                                                          int N, int T, int C4, int V) {
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= C4) return;
  for (int n0 = blockIdx.x * 4; n0 < N; n0 += gridDim.x * 4) {
    float4 a[4], p[4];
    int id[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int n = n0 + u;
      id[u] = n < N ? tok[n] : 0;
      const bool valid = n < N && id[u] >= 0 && id[u] < V;
      if (valid) {
        a[u] = __ldg(wte + (long long)id[u] * C4 + c);
        p[u] = __ldg(wpe + (long long)(n % T) * C4 + c);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int n = n0 + u;
      if (n >= N) break;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (id[u] < 0 || id[u] >= V) {
        if (c == 0) raise_device_error(DEVERR_TOKEN);
      } else {
        o = make_float4(a[u].x + p[u].x, a[u].y + p[u].y, a[u].z + p[u].z, a[u].w + p[u].w);
      }
      x[(long long)n * C4 + c] = o;
    }
  }
}

// ================================================================ LayerNorm
// y = (x - mean) * rstd * w + b over the C channels of a row; biased variance, eps 1e-5
// (nn.LayerNorm defaults, L9 "Code you'll write": Block).  One warp per row; lane l
// owns channels l + 32k, so every load and store of the warp is one coalesced line.
template <typename OutT, int CPL>
__global__ void __launch_bounds__(256) ln_fwd_kernel(const float* __restrict__ x, const float* __restrict__ w,
                                                     const float* __restrict__ b, OutT* __restrict__ y,
                                                     float* __restrict__ mean, float* __restrict__ rstd, int N) {
  constexpr int C = CPL * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= N) return;
  const float* xr = x + (long long)row * C;
  float v[CPL];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    v[k] = xr[lane + 32 * k];
    s += v[k];
  }
  const float mu = warp_sum(s) * (1.0f / C);
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    const float d = v[k] - mu;
    ss += d * d;
  }
  const float r = rsqrtf(warp_sum(ss) * (1.0f / C) + 1e-5f);
  OutT* yr = y + (long long)row * C;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    const int c = lane + 32 * k;
    st_f(yr + c, (v[k] - mu) * r * w[c] + b[c]);
  }
  if (lane == 0) {
    mean[row] = mu;
    rstd[row] = r;
  }
}

// dx = rstd * (dxhat - mean(dxhat) - xhat * mean(dxhat * xhat)),  dxhat = dy * w;
// dres = (accumulate ? dres : 0) + dx, also written in the activation type for the next
// GEMM.  Column sums accumulated in each warp's own shared-memory slice, in a fixed row
// order (block b, warp w owns rows b*8+w + k*gridDim*8), then over the 8 warps in order
// into one partial per block:  dw = sum dy * xhat,  db = sum dy,  and the sum of the new
// dres rows, which is the bias gradient of the Linear layer whose output this residual
// stream position receives (attn.c_proj or mlp.c_proj).
template <typename ActT, int CPL>
__global__ void __launch_bounds__(256, 2) ln_bwd_kernel(const ActT* __restrict__ dy, const float* __restrict__ x,
                                                        const float* __restrict__ mean, const float* __restrict__ rstd,
                                                        const float* __restrict__ w, float* __restrict__ dres,
                                                        ActT* __restrict__ dres_act, int accumulate,
                                                        float* __restrict__ part, int N) {
  constexpr int C = CPL * 32;
  extern __shared__ float red[];   // [8][3C]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* mine = red + warp * 3 * C;
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    mine[lane + 32 * k] = 0.f;
    mine[C + lane + 32 * k] = 0.f;
    mine[2 * C + lane + 32 * k] = 0.f;
  }
  for (int row = blockIdx.x * 8 + warp; row < N; row += gridDim.x * 8) {
    const ActT* dyr = dy + (long long)row * C;
    const float* xr = x + (long long)row * C;
    float* dr = dres + (long long)row * C;
    const float mu = mean[row], r = rstd[row];
    float g[CPL], xh[CPL], prev[CPL];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) prev[k] = accumulate ? dr[lane + 32 * k] : 0.f;   // issued early
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int c = lane + 32 * k;
      const float d = ld_f(dyr + c);
      xh[k] = (xr[c] - mu) * r;
      g[k] = d * __ldg(w + c);
      s1 += g[k];
      s2 += g[k] * xh[k];
      mine[c] += d * xh[k];
      mine[C + c] += d;
    }
    s1 = warp_sum(s1) * (1.0f / C);
    s2 = warp_sum(s2) * (1.0f / C);
    ActT* da = dres_act + (long long)row * C;
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int c = lane + 32 * k;
      const float o = r * (g[k] - s1 - xh[k] * s2) + prev[k];
      dr[c] = o;
      st_f(da + c, o);
      mine[2 * C + c] += o;
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 3 * C; c += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) s += red[wi * 3 * C + c];
    part[(long long)blockIdx.x * 3 * C + c] = s;
  }
}

// ================================================================ bias gradients
// out[n] += sum_m x[m, n] (bias gradients), in a fixed order: partial sums over row chunks,
// then the chunks added in order.
// Row-contiguous partial column sums: block b sums rows [b rpc, (b + 1) rpc) of every column.
// A thread owns one 16-byte group of columns (8 bf16 or 4 fp32), reads it down the rows with
// 8 loads in flight and adds the rows in order; whole rows are read by the block, so DRAM
// sees contiguous lines.
template <typename T>
__global__ void __launch_bounds__(1024) colsum_rows_kernel(const T* __restrict__ x, long long ldx, int M, int N,
                                                           int rpc, float* __restrict__ part) {
  constexpr int VEC = 16 / (int)sizeof(T);
  const int G = N / VEC;
  const int m0 = blockIdx.x * rpc, m1 = min(M, m0 + rpc);
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    float s[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) s[i] = 0.f;
    const T* p = x + (long long)m0 * ldx + g * VEC;
    auto add = [&](const uint4& q) {
      if (sizeof(T) == 2) {
        const uint32_t* u = reinterpret_cast<const uint32_t*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = unpack_bf16x2(u[i]);
          s[2 * i] += f.x;
          s[2 * i + 1] += f.y;
        }
      } else {
        const float* f = reinterpret_cast<const float*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] += f[i];
      }
    };
    int m = m0;
    for (; m + 8 <= m1; m += 8) {
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = __ldcs(reinterpret_cast<const uint4*>(p + (long long)(m - m0 + u) * ldx));
#pragma unroll
      for (int u = 0; u < 8; ++u) add(q[u]);
    }
    for (; m < m1; ++m) add(__ldcs(reinterpret_cast<const uint4*>(p + (long long)(m - m0) * ldx)));
#pragma unroll
    for (int i = 0; i < VEC; ++i) part[(long long)blockIdx.x * N + g * VEC + i] = s[i];
  }
}
// out[n] += sum_k part[k * ld + n] (k < rows, n < ncols) in a fixed order.  Block: 32 columns
// x 32 row groups; group g adds rows g, g + 32, ... in order (8 loads in flight: one batch for
// up to 256 rows), then the 32 group sums are added in group order, so the result does not
// depend on timing.
constexpr int CSR_GROUPS = 32;
__device__ __forceinline__ void colsum_fixed_order(const float* __restrict__ part, long long ld, int rows, int ncols,
                                                   int col0, float* __restrict__ out) {
  __shared__ float red[CSR_GROUPS][33];
  const int lane = threadIdx.x & 31, gr = threadIdx.x >> 5;
  const int n = col0 + lane;
  float s = 0.f;
  if (n < ncols) {
    for (int k0 = gr; k0 < rows; k0 += CSR_GROUPS * 8) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = k0 + CSR_GROUPS * i;
        v[i] = (k < rows) ? part[(long long)k * ld + n] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) s += v[i];
    }
  }
  red[gr][lane] = s;
  __syncthreads();
  if (gr == 0 && n < ncols) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < CSR_GROUPS; ++i) t += red[i][lane];
    out[n] += t;
  }
}
__global__ void __launch_bounds__(32 * CSR_GROUPS) colsum_reduce_kernel(const float* __restrict__ part, int nchunks,
                                                                       int N, float* __restrict__ out) {
  colsum_fixed_order(part, N, nchunks, N, blockIdx.x * 32, out);
}
// Many independent reductions in one launch (the gradients of the LayerNorm parameters and of
// the biases, whose partial rows the backward leaves behind): job j owns blocks
// [block0[j], block0[j + 1]).  The table is a kernel parameter, read in place.
constexpr int CSB_MAX_JOBS = 100;
struct ColsumBatchArgs {
  ColsumJob job[CSB_MAX_JOBS];
  int block0[CSB_MAX_JOBS + 1];
  int njobs;
};
static_assert(sizeof(ColsumBatchArgs) <= 4000, "kernel parameters are limited to 4 KB");
// With 16-byte accesses (columns, row stride and pointers are 16-byte multiples): a block
// takes 128 columns of one job (a float4 per lane) x 16 row groups; group g adds rows g,
// g + 16, ... in order (8 loads in flight), then the 16 group sums are added in group order,
// so the result does not depend on timing.  Blocks this wide keep HBM busy where 32-column
// blocks of 6 us each were latency-bound.
constexpr int CSB4_GROUPS = 16;
__global__ void __launch_bounds__(32 * CSB4_GROUPS) colsum_batch4_kernel(const __grid_constant__ ColsumBatchArgs a) {
  __shared__ float4 red[CSB4_GROUPS][32];
  const int bx = blockIdx.x;
  int lo = 0, hi = a.njobs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.block0[mid] <= bx) lo = mid;
    else hi = mid - 1;
  }
  const ColsumJob& j = a.job[lo];
  const int lane = threadIdx.x & 31, gr = threadIdx.x >> 5;
  const int n = (bx - a.block0[lo]) * 128 + 4 * lane;
  const int rows = j.rows;
  const long long ld = j.ld;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (n < j.ncols) {
    const float* p = j.part + n;
    for (int k0 = gr; k0 < rows; k0 += CSB4_GROUPS * 8) {
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = k0 + CSB4_GROUPS * i;
        v[i] = (k < rows) ? __ldcs(reinterpret_cast<const float4*>(p + k * ld)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        s.x += v[i].x;
        s.y += v[i].y;
        s.z += v[i].z;
        s.w += v[i].w;
      }
    }
  }
  red[gr][lane] = s;
  __syncthreads();
  if (gr == 0 && n < j.ncols) {
    float4 t = red[0][lane];
#pragma unroll
    for (int i = 1; i < CSB4_GROUPS; ++i) {
      const float4 u = red[i][lane];
      t.x += u.x;
      t.y += u.y;
      t.z += u.z;
      t.w += u.w;
    }
    float4* o = reinterpret_cast<float4*>(j.out + n);
    float4 c = *o;
    c.x += t.x;
    c.y += t.y;
    c.z += t.z;
    c.w += t.w;
    *o = c;
  }
}

// ================================================================ cross-entropy
// Combines the per-(row, column-tile) partials of the fused lm_head epilogue:
// lse = log sum_v exp(z_v) over all padded columns (L9 "2:06:39 – 2:14:58": pad rows are
// live output logits); loss_row = lse - z[target] (F.cross_entropy, L9 "52:38 – 1:06:18");
// argmax = lowest column reaching the row maximum.  Target -1 is ignored.
__device__ __forceinline__ void lse_combine(float& m, float& s, float om, float os) {
  const float nm = fmaxf(m, om);
  if (nm == -INFINITY) return;
  s = s * __expf(m - nm) + os * __expf(om - nm);
  m = nm;
}
__device__ __forceinline__ void amax_combine(float& av, int& ai, float ov, int oi) {
  if (ov > av || (ov == av && oi < ai)) {
    av = ov;
    ai = oi;
  }
}

__global__ void ce_finalize_kernel(const CePartial* __restrict__ part, int n_tiles, const float* __restrict__ zt,
                                   const int* __restrict__ targets, int N, int V, float* __restrict__ lse,
                                   float* __restrict__ loss_row, int* __restrict__ argmax) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= N) return;
  float m = -INFINITY, s = 0.f, av = -INFINITY;
  int ai = 0x7fffffff;
  for (int t = lane; t < n_tiles; t += 32) {
    const CePartial p = part[(long long)row * n_tiles + t];
    lse_combine(m, s, p.max, p.sum);
    amax_combine(av, ai, p.amax, p.aidx);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o), os = __shfl_xor_sync(0xffffffffu, s, o);
    const float oav = __shfl_xor_sync(0xffffffffu, av, o);
    const int oai = __shfl_xor_sync(0xffffffffu, ai, o);
    lse_combine(m, s, om, os);
    amax_combine(av, ai, oav, oai);
  }
  if (lane == 0) {
    const float l = m + logf(s);
    const int y = targets[row];
    const bool valid = (y >= 0 && y < V);
    if (!valid && y != -1) raise_device_error(DEVERR_TARGET);
    lse[row] = l;
    loss_row[row] = valid ? (l - zt[row]) : 0.f;
    argmax[row] = ai;
  }
}

// fp32 parity mode: the same quantities straight from an fp32 logits row.
__global__ void __launch_bounds__(256) ce_rowwise_kernel(const float* __restrict__ logits, long long ld,
                                                         const int* __restrict__ targets, int N, int Vp, int V,
                                                         float* __restrict__ lse, float* __restrict__ loss_row,
                                                         int* __restrict__ argmax) {
  __shared__ float sm[8], ss[8], sav[8];
  __shared__ int sai[8];
  const int row = blockIdx.x;
  const float* z = logits + (long long)row * ld;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = -INFINITY, s = 0.f, av = -INFINITY;
  int ai = 0x7fffffff;
  for (int v = threadIdx.x; v < Vp; v += blockDim.x) {
    const float x = z[v];
    lse_combine(m, s, x, 1.0f);
    amax_combine(av, ai, x, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o), os = __shfl_xor_sync(0xffffffffu, s, o);
    const float oav = __shfl_xor_sync(0xffffffffu, av, o);
    const int oai = __shfl_xor_sync(0xffffffffu, ai, o);
    lse_combine(m, s, om, os);
    amax_combine(av, ai, oav, oai);
  }
  if (lane == 0) {
    sm[warp] = m; ss[warp] = s; sav[warp] = av; sai[warp] = ai;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int wi = 1; wi < 8; ++wi) {
      lse_combine(m, s, sm[wi], ss[wi]);
      amax_combine(av, ai, sav[wi], sai[wi]);
    }
    const float l = m + logf(s);
    const int y = targets[row];
    const bool valid = (y >= 0 && y < V);
    if (!valid && y != -1) raise_device_error(DEVERR_TARGET);
    lse[row] = l;
    loss_row[row] = valid ? (l - z[y < 0 ? 0 : y]) : 0.f;
    argmax[row] = ai;
  }
}

// loss = mean of loss_row over valid rows (fixed-order double sum); dz_scale =
// grad_scale / count, grad_scale = 1 / grad_accum_steps (L9 "2:34:49 – 2:46:43").
__global__ void __launch_bounds__(1024) loss_reduce_kernel(const float* __restrict__ loss_row,
                                                           const int* __restrict__ targets, int N, float grad_scale,
                                                           float* loss_out, float* dz_scale_out, int* count_out) {
  __shared__ double sd[1024];
  __shared__ int sc[1024];
  double s = 0.0;
  int c = 0;
  for (int i = threadIdx.x; i < N; i += 1024) {
    s += (double)loss_row[i];
    c += (targets[i] != -1) ? 1 : 0;
  }
  sd[threadIdx.x] = s;
  sc[threadIdx.x] = c;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) {
      sd[threadIdx.x] += sd[threadIdx.x + o];
      sc[threadIdx.x] += sc[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int cnt = sc[0];
    *loss_out = cnt > 0 ? (float)(sd[0] / cnt) : 0.f;
    *dz_scale_out = cnt > 0 ? grad_scale / (float)cnt : 0.f;
    *count_out = cnt;
  }
}

// In place: z[row, v] <- (exp(z - lse) - [v == y]) * scale on valid rows, 0 on ignored rows.
template <typename T>
__global__ void ce_dz_kernel(T* __restrict__ z, long long ld, const float* __restrict__ lse,
                             const int* __restrict__ targets, const float* __restrict__ dz_scale, int Vp) {
  const int row = blockIdx.y;
  const int y = targets[row];
  const float l = lse[row];
  const float sc = (y >= 0) ? *dz_scale : 0.f;
  T* zr = z + (long long)row * ld;
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < Vp; v += gridDim.x * blockDim.x) {
    const float p = expf(ld_f(zr + v) - l);
    st_f(zr + v, (p - (v == y ? 1.f : 0.f)) * sc);
  }
}
// Persistent over rows (a grid sized to the SM count; block b takes rows b, b + grid, ...):
// each thread keeps four 16-byte streaming loads in flight.  exp(z - lse) is computed as
// 2^(z log2e - lse log2e) with the hardware ex2 (the result is rounded to bf16).
__global__ void __launch_bounds__(512) ce_dz_bf16x8_kernel(uint4* __restrict__ z, long long ld8,
                                                           const float* __restrict__ lse,
                                                           const int* __restrict__ targets,
                                                           const float* __restrict__ dz_scale, int Vp8, int N) {
  const float LOG2E = 1.4426950408889634f;
  const float scale = *dz_scale;
  for (int row = blockIdx.x; row < N; row += gridDim.x) {
    const int y = targets[row];
    const float nl = -lse[row] * LOG2E;
    const float sc = (y >= 0) ? scale : 0.f;
    uint4* zr = z + (long long)row * ld8;
    for (int i0 = threadIdx.x; i0 < Vp8; i0 += 4 * blockDim.x) {
      uint4 q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < Vp8) q[u] = __ldcs(zr + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i >= Vp8) continue;
        uint32_t* w = reinterpret_cast<uint32_t*>(&q[u]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = unpack_bf16x2(w[k]);
          const int v0 = i * 8 + 2 * k;
          const float a = (ex2(fmaf(f.x, LOG2E, nl)) - (v0 == y ? 1.f : 0.f)) * sc;
          const float bq = (ex2(fmaf(f.y, LOG2E, nl)) - (v0 + 1 == y ? 1.f : 0.f)) * sc;
          w[k] = pack_bf16x2(a, bq);
        }
        __stcs(zr + i, q[u]);
      }
    }
  }
}

// ================================================================ encoder backward
// dwte[v] += sum of dx0 rows at positions holding token v; dwpe[t] += sum_b dx0[b, t]
// (L9, "Code you'll write": wte and wpe receive the gradient of the residual stream at
// the first block's input; wte's share adds to the lm_head's, the weight being tied).
// Deterministic, with no atomics.  The (token, position) keys are put in order in two steps:
// CTAs sort segments of at most ENC_SEG consecutive positions each, then every key finds its
// place in the whole order by binary searches in the other segments (a merge by ranks).  Runs
// of equal tokens are summed in position order inside fixed ENC_CHUNK-entry chunks; a run that
// crosses chunk boundaries is finished by the chunk where it starts, which adds the later
// chunks' partial sums through eight interleaved accumulators combined in a fixed order.
constexpr int ENC_CHUNK = 32;
constexpr int ENC_SORT_THREADS = 1024;
constexpr int ENC_SEG = 4096;        // positions per sorted segment (4 keys per thread)
constexpr int ENC_SEG_BITS = 12;     // a position inside a segment
constexpr int ENC_MAX_TOKENS = 1 << (32 - ENC_SEG_BITS);   // ids below 2^20 in a segment key

// whole-order keys: token << 32 | position
__device__ __forceinline__ int key_tok(uint64_t k) { return static_cast<int>(k >> 32); }
__device__ __forceinline__ int key_pos(uint64_t k) { return static_cast<int>(k & 0xFFFFFFFFull); }
// one spare word after every 32, so that a warp reading E consecutive keys per lane
// (E a power of two up to 32) hits 32 distinct banks
__device__ __forceinline__ int enc_pad(int i) { return i + (i >> 5); }

// Compare-exchange at register distance J inside one thread's E keys; base is the
// thread's first key index, k the size of the bitonic sequences being merged.
template <int J, int E>
__device__ __forceinline__ void enc_reg_stage(uint32_t (&r)[E], int base, int k) {
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if ((e & J) == 0) {
      const uint32_t a = r[e], b = r[e | J];
      const uint32_t lo = min(a, b), hi = max(a, b);
      const bool asc = ((base + e) & k) == 0;
      r[e] = asc ? lo : hi;
      r[e | J] = asc ? hi : lo;
    }
  }
}
template <int E>
__device__ __forceinline__ void enc_reg_stages(uint32_t (&r)[E], int base, int j, int k) {
  if constexpr (E > 16) if (j == 16) enc_reg_stage<16>(r, base, k);
  if constexpr (E > 8) if (j == 8) enc_reg_stage<8>(r, base, k);
  if constexpr (E > 4) if (j == 4) enc_reg_stage<4>(r, base, k);
  if constexpr (E > 2) if (j == 2) enc_reg_stage<2>(r, base, k);
  if constexpr (E > 1) if (j == 1) enc_reg_stage<1>(r, base, k);
}

// Bitonic sort of one segment: CTA s takes positions [sP, sP + P), P = 1024 E <= ENC_SEG
// (tokens clamped to [0, V), key = token << 12 | position - sP; 0xFFFFFFFF past N) and writes
// the segment's keys in order to seg_keys[sP ..].  Thread t keeps keys tE .. tE + E-1 in
// registers: a compare-exchange at distance j < E stays in the thread, E <= j < 32E is one
// warp shuffle per key, and only the longer distances go through shared memory.
template <int E>
__global__ void __launch_bounds__(ENC_SORT_THREADS) enc_sort_kernel(const int* __restrict__ tok, int N, int V,
                                                                     uint32_t* __restrict__ seg_keys) {
  constexpr int P = ENC_SORT_THREADS * E;
  static_assert(P <= ENC_SEG, "segment larger than its position field");
  extern __shared__ uint32_t s[];   // enc_pad(P) words
  const int tid = threadIdx.x;
  const int p0 = blockIdx.x * P;
  const int n = min(P, N - p0);
  for (int i = tid; i < P; i += ENC_SORT_THREADS) {
    uint32_t key = 0xFFFFFFFFu;
    if (i < n) {
      int t = tok[p0 + i];
      t = t < 0 ? 0 : (t >= V ? V - 1 : t);
      key = (static_cast<uint32_t>(t) << ENC_SEG_BITS) | static_cast<uint32_t>(i);
    }
    s[enc_pad(i)] = key;
  }
  __syncthreads();
  const int base = tid * E;
  uint32_t r[E];
#pragma unroll
  for (int e = 0; e < E; ++e) r[e] = s[enc_pad(base + e)];
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < E) {
        enc_reg_stages<E>(r, base, j, k);
        continue;
      }
      // the partner of key i is i ^ j, in the same register slot of thread tid ^ (j / E);
      // key i keeps the smaller of the two when it is the lower index of an ascending pair
      // or the upper index of a descending one
      const bool keep_min = ((base & j) == 0) == ((base & k) == 0);
      if (j < 32 * E) {
        const int lane_dist = j / E;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint32_t b = __shfl_xor_sync(0xffffffffu, r[e], lane_dist);
          r[e] = keep_min ? min(r[e], b) : max(r[e], b);
        }
      } else {
        __syncthreads();   // every read of the previous shared-memory stage is done
#pragma unroll
        for (int e = 0; e < E; ++e) s[enc_pad(base + e)] = r[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint32_t b = s[enc_pad((base + e) ^ j)];
          r[e] = keep_min ? min(r[e], b) : max(r[e], b);
        }
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e) s[enc_pad(base + e)] = r[e];
  __syncthreads();
  for (int i = tid; i < n; i += ENC_SORT_THREADS) seg_keys[p0 + i] = s[enc_pad(i)];
}

// Merge by ranks: the key at index i of segment s (segment size P) goes to index i + (keys of
// every earlier segment with a token <= its token) + (keys of every later segment with a
// token < its token).  Equal tokens thus keep segment order, and inside a segment position
// order, so the whole is the stable (token, position) order.  One thread per key.
__global__ void __launch_bounds__(256) enc_merge_kernel(const uint32_t* __restrict__ seg_keys, int N, int P,
                                                        int nseg, uint64_t* __restrict__ sorted) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int s = i / P;
  const uint32_t key = seg_keys[i];
  const uint32_t t = key >> ENC_SEG_BITS;
  long long dst = i - (long long)s * P;
  for (int s2 = 0; s2 < nseg; ++s2) {
    if (s2 == s) continue;
    const uint32_t* a = seg_keys + (long long)s2 * P;
    const int n2 = min(P, N - s2 * P);
    const uint32_t bound = (s2 < s ? t + 1 : t) << ENC_SEG_BITS;   // count the keys below it
    int lo = 0, hi = n2;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a + mid) < bound) lo = mid + 1;
      else hi = mid;
    }
    dst += lo;
  }
  const uint32_t pos = static_cast<uint32_t>(s * P) + (key & ((1u << ENC_SEG_BITS) - 1));
  sorted[dst] = (static_cast<uint64_t>(t) << 32) | pos;
}

// One block per chunk of ENC_CHUNK sorted keys; thread x sums channels 4x .. 4x+3 of the
// chunk's rows, eight rows in flight.  A segment (the part of a run inside the chunk) that
// is a whole run goes straight into dwte; otherwise it is stored as the chunk's partial:
// slot 0 for the segment at the chunk's start, slot 1 for a run that starts later and
// leaves through the chunk's end.
__global__ void __launch_bounds__(256) enc_chunk_kernel(const uint64_t* __restrict__ sorted,
                                                        const float* __restrict__ dx0, float* __restrict__ dwte,
                                                        float* __restrict__ part, int N, int C) {
  __shared__ int tk[ENC_CHUNK + 2];   // tk[1 + i]: token of the chunk's i-th key; tk[0], tk[n + 1]: neighbours or -1
  __shared__ int ps[ENC_CHUNK];
  const int c = blockIdx.x;
  const int i0 = c * ENC_CHUNK, n = min(N - i0, ENC_CHUNK);
  for (int x = threadIdx.x; x < ENC_CHUNK + 2; x += blockDim.x) {   // blocks may have only 32 threads
    const int i = i0 - 1 + x;
    int t = -1;
    if (i >= 0 && i < N && x <= n + 1) {
      const uint64_t key = sorted[i];
      t = key_tok(key);
      if (x >= 1 && x <= n) ps[x - 1] = key_pos(key);
    }
    tk[x] = t;
  }
  __syncthreads();
  const int ch = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (ch >= C) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int seg_start = 0;
  for (int g = 0; g < n; g += 8) {
    float4 d[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (g + u < n) d[u] = __ldg(reinterpret_cast<const float4*>(dx0 + (long long)ps[g + u] * C + ch));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = g + u;
      if (i >= n) break;
      acc.x += d[u].x; acc.y += d[u].y; acc.z += d[u].z; acc.w += d[u].w;
      const int t = tk[i + 1];
      const bool run_end = tk[i + 2] != t;
      if (run_end || i + 1 == n) {
        const bool starts_here = seg_start > 0 || tk[0] != t;
        if (starts_here && run_end) {
          float4* o = reinterpret_cast<float4*>(dwte + (long long)t * C + ch);
          float4 w = *o;
          w.x += acc.x; w.y += acc.y; w.z += acc.z; w.w += acc.w;
          *o = w;
        } else {
          const int slot = seg_start == 0 ? 0 : 1;
          *reinterpret_cast<float4*>(part + ((long long)c * 2 + slot) * C + ch) = acc;
        }
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        seg_start = i + 1;
      }
    }
  }
}

// The chunk where a boundary-crossing run starts adds its own partial and, over eight
// interleaved accumulators (chunk c + 1 + q goes to accumulator q mod 8, each in chunk
// order, then accumulators 0..7 in turn), slot 0 of every later chunk the run covers.
__global__ void __launch_bounds__(256) enc_fixup_kernel(const uint64_t* __restrict__ sorted,
                                                        float* __restrict__ dwte, const float* __restrict__ part,
                                                        int N, int C, int nchunks) {
  __shared__ int last_chunk;
  const int c = blockIdx.x;
  const int i0 = c * ENC_CHUNK, i1 = min(N, i0 + ENC_CHUNK);
  const int t = key_tok(sorted[i1 - 1]);
  const bool crosses_out = (i1 < N) && key_tok(sorted[i1]) == t;
  const bool crosses_in = (i0 > 0) && key_tok(sorted[i0 - 1]) == t && key_tok(sorted[i0]) == t;
  if (!crosses_out || crosses_in) return;
  if (threadIdx.x < 32) {
    // the run's last chunk: one before the first later chunk that starts with another
    // token (or the end), looked up 32 chunk heads per ballot; chunk c + 1 starts with t
    int c_last = -1;
    for (int cb = c + 1; c_last < 0; cb += 32) {
      const int cc = cb + static_cast<int>(threadIdx.x);
      const bool other = cc >= nchunks || key_tok(sorted[(long long)cc * ENC_CHUNK]) != t;
      const unsigned m = __ballot_sync(0xffffffffu, other);
      if (m) c_last = cb + __ffs(m) - 2;
    }
    if (threadIdx.x == 0) last_chunk = c_last;
  }
  __syncthreads();
  const int ch = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (ch >= C) return;
  const int slot = key_tok(sorted[i0]) == t ? 0 : 1;
  const int cnt = last_chunk - c;
  float4 a[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int q0 = 0; q0 < cnt; q0 += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (q0 + u < cnt) {
        const float4 p = __ldg(reinterpret_cast<const float4*>(part + (long long)(c + 1 + q0 + u) * 2 * C + ch));
        a[u].x += p.x; a[u].y += p.y; a[u].z += p.z; a[u].w += p.w;
      }
    }
  }
  float4 tot = *reinterpret_cast<const float4*>(part + ((long long)c * 2 + slot) * C + ch);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    tot.x += a[u].x; tot.y += a[u].y; tot.z += a[u].z; tot.w += a[u].w;
  }
  float4* o = reinterpret_cast<float4*>(dwte + (long long)t * C + ch);
  float4 w = *o;
  w.x += tot.x; w.y += tot.y; w.z += tot.z; w.w += tot.w;
  *o = w;
}

// ================================================================ top-k sampling
// Next-token sampling from rows of logits (L9, "28:07 – 41:44 Loading the weights and
// generating text"): the k largest logits, ties to the lower id, in descending order, their
// softmax, and the inverse CDF at the caller's uniform.  One CTA per sampled row.  Round r
// takes the block-wide maximum of the composite keys (order-preserving logit bits, then the
// complemented id) below round r-1's winner, so the kept list comes out already ordered,
// with nothing marked and nothing sorted.  Not on the training step's path.
constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_MAX = 1024;

// a < b  <=>  topk_order_bits(a) < topk_order_bits(b) for every non-NaN float
__device__ __forceinline__ uint32_t topk_order_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float topk_load(const float* p) { return __ldg(p); }
__device__ __forceinline__ float topk_load(const bf16* p) { return __bfloat162float(*p); }

template <typename T>
__global__ void __launch_bounds__(TOPK_THREADS) topk_sample_kernel(const T* __restrict__ logits, long long ld,
                                                                   int n_rows, const int* __restrict__ rows,
                                                                   const float* __restrict__ u, int V, int k,
                                                                   int* __restrict__ out, int* __restrict__ out_topk) {
  __shared__ unsigned long long warp_best[TOPK_THREADS / 32];
  __shared__ unsigned long long best;
  __shared__ int sel[TOPK_MAX];
  __shared__ float selv[TOPK_MAX];
  const int s = blockIdx.x;
  const int row = rows[s];
  if (row < 0 || row >= n_rows) {   // the same for the whole block
    if (threadIdx.x == 0) {
      out[s] = -1;
      raise_device_error(DEVERR_ROW);
    }
    if (out_topk)
      for (int j = threadIdx.x; j < k; j += TOPK_THREADS) out_topk[(long long)s * k + j] = -1;
    return;
  }
  const T* z = logits + (long long)row * ld;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned long long limit = ~0ull;
  for (int r = 0; r < k; ++r) {
    unsigned long long mine = 0;
    for (int i = threadIdx.x; i < V; i += TOPK_THREADS) {
      const unsigned long long key = (static_cast<unsigned long long>(topk_order_bits(topk_load(z + i))) << 32) |
                                     static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(i));
      if ((r == 0 || key < limit) && key > mine) mine = key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, mine, o);
      mine = other > mine ? other : mine;
    }
    if (lane == 0) warp_best[warp] = mine;
    __syncthreads();
    if (warp == 0) {
      mine = warp_best[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, mine, o);
        mine = other > mine ? other : mine;
      }
      if (lane == 0) {
        best = mine;
        const int id = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(mine & 0xFFFFFFFFull));
        sel[r] = id;
        selv[r] = topk_load(z + id);
      }
    }
    __syncthreads();
    limit = best;
  }
  if (out_topk)
    for (int j = threadIdx.x; j < k; j += TOPK_THREADS) out_topk[(long long)s * k + j] = sel[j];
  if (threadIdx.x == 0) {
    // softmax over the kept logits relative to the largest, summed in the kept order
    float total = 0.f;
    for (int j = 0; j < k; ++j) total += expf(selv[j] - selv[0]);
    float uu = u[s];
    uu = (uu >= 0.f) ? uu : 0.f;
    uu = (uu < 1.f) ? uu : 0.99999994f;
    const float target = uu * total;
    float cum = 0.f;
    int pick = sel[k - 1];
    for (int j = 0; j < k; ++j) {
      cum += expf(selv[j] - selv[0]);
      if (cum > target) {
        pick = sel[j];
        break;
      }
    }
    out[s] = pick;
  }
}

// dwpe[t] += sum over b in order of dx0[b, t]: four channels per thread, eight rows in flight.
__global__ void __launch_bounds__(256) dwpe_kernel(const float4* __restrict__ dx0, float4* __restrict__ dwpe, int B,
                                                   int TC4) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < TC4; i += gridDim.x * blockDim.x) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int b0 = 0; b0 < B; b0 += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (b0 + u < B) v[u] = __ldg(dx0 + (long long)(b0 + u) * TC4 + i);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (b0 + u < B) {
          s.x += v[u].x; s.y += v[u].y; s.z += v[u].z; s.w += v[u].w;
        }
      }
    }
    float4 w = dwpe[i];
    w.x += s.x; w.y += s.y; w.z += s.z; w.w += s.w;
    dwpe[i] = w;
  }
}

// ================================================================ norm, AdamW, init
// Global gradient norm sqrt(sum g^2) (L9 "2:14:58 – 2:25:57": clip_grad_norm_ at 1.0),
// fixed grid and fixed-order double partials; scale = min(1, clip / (norm + 1e-6)).
__global__ void __launch_bounds__(512) sumsq_kernel(const float* __restrict__ g, long long n,
                                                    double* __restrict__ part) {
  __shared__ double sd[512];
  // four independent 16-byte loads in flight per thread, each squared in fp32 and summed in
  // double along its own chain; the chains and then the threads are added in a fixed order
  double s4[4] = {0.0, 0.0, 0.0, 0.0};
  const long long n4 = n / 4;
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const long long stride = (long long)gridDim.x * 512;
  long long i = blockIdx.x * 512LL + threadIdx.x;
  for (; i + 3 * stride < n4; i += 4 * stride) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(g4 + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      s4[u] += (double)(v[u].x * v[u].x) + (double)(v[u].y * v[u].y) + (double)(v[u].z * v[u].z) +
               (double)(v[u].w * v[u].w);
  }
  for (; i < n4; i += stride) {
    const float4 v = __ldcs(g4 + i);
    s4[0] += (double)(v.x * v.x) + (double)(v.y * v.y) + (double)(v.z * v.z) + (double)(v.w * v.w);
  }
  double s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  if (blockIdx.x == 0)
    for (long long j = n4 * 4 + threadIdx.x; j < n; j += 512) s += (double)g[j] * (double)g[j];
  sd[threadIdx.x] = s;
  __syncthreads();
  for (int o = 256; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) sd[threadIdx.x] += sd[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = sd[0];
}
__global__ void norm_finalize_kernel(const double* __restrict__ part, int nparts, float clip, float* out2) {
  __shared__ double sd[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < nparts; i += 256) s += part[i];
  sd[threadIdx.x] = s;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) sd[threadIdx.x] += sd[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double norm = sqrt(sd[0]);
    out2[0] = (float)norm;
    out2[1] = (float)fmin(1.0, (double)clip / (norm + 1e-6));
  }
}

// AdamW with decoupled weight decay and bias correction (torch.optim.AdamW semantics; L9
// "2:14:58 – 2:25:57" betas/eps, "2:25:57 – 2:34:49" decay on >= 2-D tensors only).
// One launch updates every tensor; each block reads its (offset, count, decay) entry.
// Blocks start on 16-byte boundaries and hold a multiple of 4 elements (every tensor size is
// a multiple of n_embd), so each thread moves 4 elements per access with 16-byte loads and
// stores, two groups in flight (p, g, m and v: eight loads).
__device__ __forceinline__ float adamw_one(float& mi, float& vi, float pi, float gi, float s, float b1, float b2,
                                           float lr, float eps, float decay, float bc1, float bc2) {
  gi *= s;
  mi = b1 * mi + (1.0f - b1) * gi;
  vi = b2 * vi + (1.0f - b2) * gi * gi;
  const float mh = mi / bc1;
  const float vh = vi / bc2;
  return pi * decay - lr * mh / (sqrtf(vh) + eps);
}
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    bf16* __restrict__ shadow, const AdamBlock* __restrict__ blocks,
                                                    const float* __restrict__ clip_scale, float lr, float b1,
                                                    float b2, float eps, float wd, float bc1, float bc2) {
  const AdamBlock blk = blocks[blockIdx.x];
  const float s = *clip_scale;
  const float decay = blk.decay ? (1.0f - lr * wd) : 1.0f;
  const bool write_shadow = shadow != nullptr && blk.decay;
  float4* p4 = reinterpret_cast<float4*>(p + blk.off);
  const float4* g4 = reinterpret_cast<const float4*>(g + blk.off);
  float4* m4 = reinterpret_cast<float4*>(m + blk.off);
  float4* v4 = reinterpret_cast<float4*>(v + blk.off);
  uint2* sh4 = reinterpret_cast<uint2*>(shadow + blk.off);
  const int n4 = blk.n >> 2;
  for (int i0 = threadIdx.x; i0 < n4; i0 += 2 * blockDim.x) {
    float4 pv[2], gv[2], mv[2], vv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < n4) {
        pv[u] = p4[i];
        gv[u] = __ldcs(g4 + i);
        mv[u] = __ldcs(m4 + i);
        vv[u] = __ldcs(v4 + i);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i >= n4) continue;
      float4 o;
      o.x = adamw_one(mv[u].x, vv[u].x, pv[u].x, gv[u].x, s, b1, b2, lr, eps, decay, bc1, bc2);
      o.y = adamw_one(mv[u].y, vv[u].y, pv[u].y, gv[u].y, s, b1, b2, lr, eps, decay, bc1, bc2);
      o.z = adamw_one(mv[u].z, vv[u].z, pv[u].z, gv[u].z, s, b1, b2, lr, eps, decay, bc1, bc2);
      o.w = adamw_one(mv[u].w, vv[u].w, pv[u].w, gv[u].w, s, b1, b2, lr, eps, decay, bc1, bc2);
      p4[i] = o;
      __stcs(m4 + i, mv[u]);
      __stcs(v4 + i, vv[u]);
      if (write_shadow) sh4[i] = make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
    }
  }
}

// Initialisation draw: value e of a tensor = float(std * sqrt(-2 ln u1) cos(2 pi u2)) with
// u1 = 1 - (r_{2e} >> 11) 2^-53, u2 = (r_{2e+1} >> 11) 2^-53, r_j the j-th SplitMix64
// output (Steele, Lea & Flood 2014) of the tensor's state.  Double-precision log, cos and
// sqrt are CUDA's, called.
__device__ __forceinline__ uint64_t splitmix64_at(uint64_t state, uint64_t j) {
  uint64_t z = state + (j + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__global__ void init_normal_kernel(float* __restrict__ p, long long n, uint64_t state, double std) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const uint64_t r1 = splitmix64_at(state, 2ull * e), r2 = splitmix64_at(state, 2ull * e + 1ull);
    const double u1 = 1.0 - (double)(r1 >> 11) * 0x1.0p-53;
    const double u2 = (double)(r2 >> 11) * 0x1.0p-53;
    const double z = sqrt(-2.0 * log(u1)) * cos(2.0 * 3.141592653589793 * u2);
    p[e] = (float)(std * z);
  }
}
__global__ void fill_kernel(float* __restrict__ p, long long n, float value) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    p[e] = value;
}
__global__ void cast_bf16_kernel(const float* __restrict__ s, bf16* __restrict__ d, long long n) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    d[e] = __float2bfloat16_rn(s[e]);
}

inline int grid_for(long long n, int threads, int cap = 148 * 16) {
  long long g = cdivll(n, threads);
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}
inline int ok() { return cudaGetLastError() == cudaSuccess ? 0 : -3; }

// Same with 16-byte accesses (C a multiple of 128): lane l holds float4 groups l, l + 32, ...;
// gamma and beta stay in registers across the rows a warp takes (rows warp, warp + stride,
// ... of a grid sized to the SM count).
template <typename OutT, int V4>
__global__ void __launch_bounds__(256) ln_fwd_vec_kernel(const float* __restrict__ x, const float* __restrict__ w,
                                                         const float* __restrict__ b, OutT* __restrict__ y,
                                                         float* __restrict__ mean, float* __restrict__ rstd, int N) {
  constexpr int C = V4 * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4 wv[V4], bv[V4];
#pragma unroll
  for (int k = 0; k < V4; ++k) {
    wv[k] = reinterpret_cast<const float4*>(w)[lane + 32 * k];
    bv[k] = reinterpret_cast<const float4*>(b)[lane + 32 * k];
  }
  // rows up to 768 columns also load the warp's next row before working on the current one,
  // so that two rows' loads are in flight (wider rows have no registers to spare for it)
  constexpr bool PREFETCH = V4 <= 6;
  const int stride = gridDim.x * 8;
  float4 nv[PREFETCH ? V4 : 1];
  int row = blockIdx.x * 8 + warp;
  if (PREFETCH && row < N) {
    const float4* xr = reinterpret_cast<const float4*>(x + (long long)row * C);
#pragma unroll
    for (int k = 0; k < V4; ++k) nv[PREFETCH ? k : 0] = __ldcs(xr + lane + 32 * k);
  }
  for (; row < N; row += stride) {
    float4 v[V4];
    if (PREFETCH) {
#pragma unroll
      for (int k = 0; k < V4; ++k) v[k] = nv[PREFETCH ? k : 0];
      if (row + stride < N) {
        const float4* xn = reinterpret_cast<const float4*>(x + (long long)(row + stride) * C);
#pragma unroll
        for (int k = 0; k < V4; ++k) nv[PREFETCH ? k : 0] = __ldcs(xn + lane + 32 * k);
      }
    } else {
      const float4* xr = reinterpret_cast<const float4*>(x + (long long)row * C);
#pragma unroll
      for (int k = 0; k < V4; ++k) v[k] = __ldcs(xr + lane + 32 * k);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < V4; ++k) s += (v[k].x + v[k].y) + (v[k].z + v[k].w);
    const float mu = warp_sum(s) * (1.0f / C);
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const float a = v[k].x - mu, bq = v[k].y - mu, c = v[k].z - mu, d = v[k].w - mu;
      ss += (a * a + bq * bq) + (c * c + d * d);
    }
    const float r = rsqrtf(warp_sum(ss) * (1.0f / C) + 1e-5f);
    OutT* yr = y + (long long)row * C;
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const float o0 = (v[k].x - mu) * r * wv[k].x + bv[k].x, o1 = (v[k].y - mu) * r * wv[k].y + bv[k].y;
      const float o2 = (v[k].z - mu) * r * wv[k].z + bv[k].z, o3 = (v[k].w - mu) * r * wv[k].w + bv[k].w;
      const int c = 4 * (lane + 32 * k);
      if (sizeof(OutT) == 2) {
        uint2 pk;
        pk.x = pack_bf16x2(o0, o1);
        pk.y = pack_bf16x2(o2, o3);
        *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(yr) + c) = pk;
      } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(yr) + c) = make_float4(o0, o1, o2, o3);
      }
    }
    if (lane == 0) {
      mean[row] = mu;
      rstd[row] = r;
    }
  }
}

template <typename OutT>
int ln_fwd_dispatch(cudaStream_t st, const float* x, const float* w, const float* b, OutT* y, float* mean,
                    float* rstd, int N, int C) {
  const int grid = cdiv(N, 8);
  // 16-byte path: x, w, b, y 16-byte aligned and C a multiple of 128
  const bool vec = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(b) |
                     reinterpret_cast<uintptr_t>(y)) % 16) == 0;
  const int nsm = current_device_sms();
  const int vgrid = grid < nsm * 2 ? grid : nsm * 2;   // 2 resident blocks per SM (registers), rows strided
  if (vec && (C == 768 || C == 1024 || C == 512 || C == 384 || C == 256 || C == 128)) {
    switch (C) {
#define LNV(V4) case V4 * 128: ln_fwd_vec_kernel<OutT, V4><<<vgrid, 256, 0, st>>>(x, w, b, y, mean, rstd, N); break;
      LNV(1) LNV(2) LNV(3) LNV(4) LNV(6) LNV(8)
#undef LNV
    }
    note_kernel_launches(1);
    return ok();
  }
  switch (C) {
#define LNF(CPL) case CPL * 32: ln_fwd_kernel<OutT, CPL><<<grid, 256, 0, st>>>(x, w, b, y, mean, rstd, N); break;
    LNF(1) LNF(2) LNF(4) LNF(8) LNF(12) LNF(16) LNF(24) LNF(32)
#undef LNF
    default: return -4;
  }
  note_kernel_launches(1);
  return ok();
}

// Same with 16-byte accesses (C a multiple of 128): lane l holds float4 column groups
// l, l + 32, ...; gamma stays in registers and the per-warp accumulators are updated four
// columns at a time.
// Four consecutive values (16-byte aligned group c4 of a row) as fp32, streaming load.
__device__ __forceinline__ float4 ld4_stream(const float* row, int c4) {
  return __ldcs(reinterpret_cast<const float4*>(row) + c4);
}
__device__ __forceinline__ float4 ld4_stream(const bf16* row, int c4) {
  const uint2 q = __ldcs(reinterpret_cast<const uint2*>(row) + c4);
  const float2 a = unpack_bf16x2(q.x), b = unpack_bf16x2(q.y);
  return make_float4(a.x, a.y, b.x, b.y);
}

template <typename ActT, int V4>
__global__ void __launch_bounds__(256, 2) ln_bwd_vec_kernel(const ActT* __restrict__ dy, const float* __restrict__ x,
                                                            const float* __restrict__ mean,
                                                            const float* __restrict__ rstd, const float* __restrict__ w,
                                                            float* __restrict__ dres, ActT* __restrict__ dres_act,
                                                            int accumulate, float* __restrict__ part, int N) {
  constexpr int C = V4 * 128, C4 = C / 4;
  extern __shared__ float red[];   // [8][3C]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* mine = reinterpret_cast<float4*>(red + warp * 3 * C);
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr bool HOIST_W = V4 <= 6;   // wider rows load gamma per row (registers)
  float4 wv[HOIST_W ? V4 : 1];
#pragma unroll
  for (int k = 0; k < V4; ++k) {
    mine[lane + 32 * k] = z4;
    mine[C4 + lane + 32 * k] = z4;
    mine[2 * C4 + lane + 32 * k] = z4;
    if (HOIST_W) wv[HOIST_W ? k : 0] = __ldg(reinterpret_cast<const float4*>(w) + lane + 32 * k);
  }
  for (int row = blockIdx.x * 8 + warp; row < N; row += gridDim.x * 8) {
    const ActT* dyr = dy + (long long)row * C;
    const float4* xr = reinterpret_cast<const float4*>(x + (long long)row * C);
    float4* dr = reinterpret_cast<float4*>(dres + (long long)row * C);
    const float mu = mean[row], r = rstd[row];
    float4 g[V4], xh[V4], prev[V4];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int k = 0; k < V4; ++k) prev[k] = accumulate ? dr[lane + 32 * k] : z4;   // issued early
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const int c = lane + 32 * k;
      const float4 d = ld4_stream(dyr, c), xv = __ldcs(xr + c);
      xh[k] = make_float4((xv.x - mu) * r, (xv.y - mu) * r, (xv.z - mu) * r, (xv.w - mu) * r);
      const float4 wk = HOIST_W ? wv[HOIST_W ? k : 0] : __ldg(reinterpret_cast<const float4*>(w) + c);
      g[k] = make_float4(d.x * wk.x, d.y * wk.y, d.z * wk.z, d.w * wk.w);
      s1 += (g[k].x + g[k].y) + (g[k].z + g[k].w);
      s2 += (g[k].x * xh[k].x + g[k].y * xh[k].y) + (g[k].z * xh[k].z + g[k].w * xh[k].w);
      float4 a = mine[c];
      a.x += d.x * xh[k].x; a.y += d.y * xh[k].y; a.z += d.z * xh[k].z; a.w += d.w * xh[k].w;
      mine[c] = a;
      float4 bb = mine[C4 + c];
      bb.x += d.x; bb.y += d.y; bb.z += d.z; bb.w += d.w;
      mine[C4 + c] = bb;
    }
    s1 = warp_sum(s1) * (1.0f / C);
    s2 = warp_sum(s2) * (1.0f / C);
    ActT* da = dres_act + (long long)row * C;
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const int c = lane + 32 * k;
      float4 o;
      o.x = r * (g[k].x - s1 - xh[k].x * s2) + prev[k].x;
      o.y = r * (g[k].y - s1 - xh[k].y * s2) + prev[k].y;
      o.z = r * (g[k].z - s1 - xh[k].z * s2) + prev[k].z;
      o.w = r * (g[k].w - s1 - xh[k].w * s2) + prev[k].w;
      dr[c] = o;
      if (sizeof(ActT) == 2) {
        uint2 pk;
        pk.x = pack_bf16x2(o.x, o.y);
        pk.y = pack_bf16x2(o.z, o.w);
        *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(da) + 4 * c) = pk;
      } else {
        reinterpret_cast<float4*>(da)[c] = o;
      }
      float4 t = mine[2 * C4 + c];
      t.x += o.x; t.y += o.y; t.z += o.z; t.w += o.w;
      mine[2 * C4 + c] = t;
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 3 * C; c += blockDim.x) {
    float sum = 0.f;
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) sum += red[wi * 3 * C + c];
    part[(long long)blockIdx.x * 3 * C + c] = sum;
  }
}

template <typename ActT>
int ln_bwd_dispatch(cudaStream_t st, const ActT* dy, const float* x, const float* mean, const float* rstd,
                    const float* w, float* dres, ActT* dres_act, int acc, float* part, int nblocks, int N, int C) {
  const int smem = 8 * 3 * C * (int)sizeof(float);
  const bool vec = ((reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(x) |
                     reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(dres) |
                     reinterpret_cast<uintptr_t>(dres_act)) % 16) == 0;
  // (fp32 activations at 1024 columns stay on the scalar path: the vector form would spill)
  const bool vec_c = C == 768 || C == 512 || C == 384 || C == 256 || C == 128 || (C == 1024 && sizeof(ActT) == 2);
  if (vec && vec_c) {
    switch (C) {
#define LNBV(V4)                                                                                                 \
  case V4 * 128: {                                                                                               \
    auto k = ln_bwd_vec_kernel<ActT, V4>;                                                                        \
    if (smem > 48 * 1024 && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) return -3; \
    k<<<nblocks, 256, smem, st>>>(dy, x, mean, rstd, w, dres, dres_act, acc, part, N);                           \
    break;                                                                                                       \
  }
      LNBV(1) LNBV(2) LNBV(3) LNBV(4) LNBV(6)
      case 8 * 128:
        if constexpr (sizeof(ActT) == 2) {
          auto k = ln_bwd_vec_kernel<ActT, 8>;
          if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) return -3;
          k<<<nblocks, 256, smem, st>>>(dy, x, mean, rstd, w, dres, dres_act, acc, part, N);
        }
        break;
#undef LNBV
    }
    note_kernel_launches(1);
    return ok();
  }
  switch (C) {
#define LNB(CPL)                                                                                               \
  case CPL * 32: {                                                                                             \
    auto k = ln_bwd_kernel<ActT, CPL>;                                                                         \
    if (smem > 48 * 1024 && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) return -3; \
    k<<<nblocks, 256, smem, st>>>(dy, x, mean, rstd, w, dres, dres_act, acc, part, N);                         \
    break;                                                                                                     \
  }
    LNB(1) LNB(2) LNB(4) LNB(8) LNB(12) LNB(16) LNB(24) LNB(32)
#undef LNB
    default: return -4;
  }
  note_kernel_launches(1);
  return ok();
}

}  // namespace

// ==================================================================== launchers
int launch_encoder_fwd(cudaStream_t st, const int* tok, const float* wte, const float* wpe, float* x, int N, int T,
                       int C, int V) {
  if (N <= 0 || T <= 0 || C <= 0 || C % 4) return -4;
  // 16-byte accesses: the tables and the output must be 16-byte aligned
  if ((reinterpret_cast<uintptr_t>(wte) | reinterpret_cast<uintptr_t>(wpe) | reinterpret_cast<uintptr_t>(x)) % 16)
    return -1;
  const int c4 = C / 4;
  const int threads = c4 <= 256 ? (c4 + 31) / 32 * 32 : 256;
  dim3 grid(grid_for(cdiv(N, 4), 1, 148 * 8), cdiv(c4, threads));
  encoder_fwd_kernel<<<grid, threads, 0, st>>>(tok, reinterpret_cast<const float4*>(wte),
                                               reinterpret_cast<const float4*>(wpe), reinterpret_cast<float4*>(x),
                                               N, T, c4, V);
  note_kernel_launches(1);
  return ok();
}

int launch_layernorm_fwd(cudaStream_t st, bool is_bf16, const float* x, const float* w, const float* b, void* y,
                         float* mean, float* rstd, int N, int C) {
  if (is_bf16) return ln_fwd_dispatch<bf16>(st, x, w, b, reinterpret_cast<bf16*>(y), mean, rstd, N, C);
  return ln_fwd_dispatch<float>(st, x, w, b, reinterpret_cast<float*>(y), mean, rstd, N, C);
}

int layernorm_bwd_blocks(int num_sms) { return 2 * num_sms; }

int launch_layernorm_bwd(cudaStream_t st, bool is_bf16, const void* dy, const float* x, const float* mean,
                         const float* rstd, const float* w, float* dres, void* dres_act, bool accumulate, float* part,
                         int nblocks, int N, int C) {
  int rc = is_bf16 ? ln_bwd_dispatch<bf16>(st, reinterpret_cast<const bf16*>(dy), x, mean, rstd, w, dres,
                                           reinterpret_cast<bf16*>(dres_act), accumulate, part, nblocks, N, C)
                   : ln_bwd_dispatch<float>(st, reinterpret_cast<const float*>(dy), x, mean, rstd, w, dres,
                                            reinterpret_cast<float*>(dres_act), accumulate, part, nblocks, N, C);
  if (rc) return rc;
  return ok();
}

// Row chunks of the column sums (a function of M only, so the partial buffer sized with it
// matches every launch): up to 256 chunks of at least 32 rows.
int colsum_chunks(int M) { return M < 32 ? 1 : (cdiv(M, 32) < 256 ? cdiv(M, 32) : 256); }

int launch_colsum(cudaStream_t st, bool is_bf16, const void* x, long long ldx, int M, int N, float* part,
                  int nchunks, float* out) {
  if (N % 8 != 0 || ldx % 8 != 0 || nchunks != colsum_chunks(M) || (reinterpret_cast<uintptr_t>(x) % 16) != 0)
    return -4;
  const int rpc = cdiv(M, nchunks);
  const int used = cdiv(M, rpc);
  const int groups = N / (is_bf16 ? 8 : 4);
  int threads = (groups + 31) / 32 * 32;
  if (threads > 1024) threads = 1024;
  if (is_bf16) colsum_rows_kernel<bf16><<<used, threads, 0, st>>>(reinterpret_cast<const bf16*>(x), ldx, M, N, rpc, part);
  else colsum_rows_kernel<float><<<used, threads, 0, st>>>(reinterpret_cast<const float*>(x), ldx, M, N, rpc, part);
  colsum_reduce_kernel<<<cdiv(N, 32), 32 * CSR_GROUPS, 0, st>>>(part, used, N, out);
  note_kernel_launches(2);
  return ok();
}

int launch_colsum_batch(cudaStream_t st, const ColsumJob* jobs, int njobs) {
  for (int j = 0; j < njobs; ++j)
    if (jobs[j].part == nullptr || jobs[j].out == nullptr || jobs[j].rows <= 0 || jobs[j].ncols <= 0 ||
        jobs[j].ld < jobs[j].ncols)
      return -4;
  for (int j = 0; j < njobs; ++j)
    if (jobs[j].ncols % 4 != 0 || jobs[j].ld % 4 != 0 || reinterpret_cast<uintptr_t>(jobs[j].part) % 16 != 0 ||
        reinterpret_cast<uintptr_t>(jobs[j].out) % 16 != 0)
      return -1;
  for (int first = 0; first < njobs; first += CSB_MAX_JOBS) {
    ColsumBatchArgs a;
    a.njobs = njobs - first < CSB_MAX_JOBS ? njobs - first : CSB_MAX_JOBS;
    int blocks = 0;
    for (int j = 0; j < a.njobs; ++j) {
      a.job[j] = jobs[first + j];
      a.block0[j] = blocks;
      blocks += cdiv(a.job[j].ncols, 128);
    }
    a.block0[a.njobs] = blocks;
    colsum_batch4_kernel<<<blocks, 32 * CSB4_GROUPS, 0, st>>>(a);
    note_kernel_launches(1);
  }
  return ok();
}

int launch_ce_finalize(cudaStream_t st, const CePartial* part, int n_tiles, const float* zt, const int* targets,
                       int N, int V, float* lse, float* loss_row, int* argmax) {
  ce_finalize_kernel<<<cdiv(N, 8), 256, 0, st>>>(part, n_tiles, zt, targets, N, V, lse, loss_row, argmax);
  note_kernel_launches(1);
  return ok();
}

int launch_ce_rowwise(cudaStream_t st, const float* logits, long long ld, const int* targets, int N, int Vp, int V,
                      float* lse, float* loss_row, int* argmax) {
  ce_rowwise_kernel<<<N, 256, 0, st>>>(logits, ld, targets, N, Vp, V, lse, loss_row, argmax);
  note_kernel_launches(1);
  return ok();
}

int launch_loss_reduce(cudaStream_t st, const float* loss_row, const int* targets, int N, float grad_scale,
                       float* loss_out, float* dz_scale_out, int* count_out) {
  loss_reduce_kernel<<<1, 1024, 0, st>>>(loss_row, targets, N, grad_scale, loss_out, dz_scale_out, count_out);
  note_kernel_launches(1);
  return ok();
}

int launch_ce_dz(cudaStream_t st, bool is_bf16, void* logits, long long ld, const float* lse, const int* targets,
                 const float* dz_scale, int N, int Vp) {
  if (is_bf16 && Vp % 8 == 0 && ld % 8 == 0) {
    const int v8 = Vp / 8;
    const int nsm = current_device_sms();
    const int grid = N < nsm * 4 ? N : nsm * 4;   // 4 blocks of 512 threads per SM
    ce_dz_bf16x8_kernel<<<grid, 512, 0, st>>>(reinterpret_cast<uint4*>(logits), ld / 8, lse, targets, dz_scale, v8,
                                              N);
  } else {
    dim3 grid(cdiv(Vp, 256), N);
    if (is_bf16) ce_dz_kernel<bf16><<<grid, 256, 0, st>>>(reinterpret_cast<bf16*>(logits), ld, lse, targets, dz_scale, Vp);
    else ce_dz_kernel<float><<<grid, 256, 0, st>>>(reinterpret_cast<float*>(logits), ld, lse, targets, dz_scale, Vp);
  }
  note_kernel_launches(1);
  return ok();
}

size_t encoder_bwd_part_floats(int N, int C) { return (size_t)cdiv(N, ENC_CHUNK) * 2 * (size_t)C; }

template <int E>
static int enc_sort_launch(cudaStream_t st, const int* tok, int N, int V, uint32_t* seg_keys) {
  constexpr int P = ENC_SORT_THREADS * E;
  const int smem = (P + P / 32) * (int)sizeof(uint32_t);
  if (smem > 48 * 1024 && set_dynamic_smem_once((const void*)enc_sort_kernel<E>, smem)) return -3;
  enc_sort_kernel<E><<<cdiv(N, P), ENC_SORT_THREADS, smem, st>>>(tok, N, V, seg_keys);
  return 0;
}

size_t encoder_bwd_seg_words(int N) { return ((size_t)N + 63) / 64 * 64; }

int launch_encoder_bwd(cudaStream_t st, const int* tok, const float* dx0, float* dwte, float* dwpe, int B, int T,
                       int C, uint64_t* sorted_keys, uint32_t* seg_keys, float* chunk_part, int V) {
  const long long Nll = (long long)B * T;
  if (B <= 0 || T <= 0 || Nll > ENC_MAX_POSITIONS || V <= 0 || V >= ENC_MAX_TOKENS || C <= 0 || C % 4) return -4;
  // 16-byte accesses to dx0, the gradients and the chunk partials
  if ((reinterpret_cast<uintptr_t>(dx0) | reinterpret_cast<uintptr_t>(dwte) | reinterpret_cast<uintptr_t>(dwpe) |
       reinterpret_cast<uintptr_t>(chunk_part)) % 16)
    return -1;
  const int N = (int)Nll;
  // one segment of 1024 E keys for short inputs, segments of ENC_SEG keys otherwise
  int P = ENC_SORT_THREADS;
  while (P < N && P < ENC_SEG) P <<= 1;
  int rc;
  switch (P / ENC_SORT_THREADS) {
    case 1: rc = enc_sort_launch<1>(st, tok, N, V, seg_keys); break;
    case 2: rc = enc_sort_launch<2>(st, tok, N, V, seg_keys); break;
    default: rc = enc_sort_launch<4>(st, tok, N, V, seg_keys); break;
  }
  if (rc) return rc;
  enc_merge_kernel<<<cdiv(N, 256), 256, 0, st>>>(seg_keys, N, P, cdiv(N, P), sorted_keys);
  const int nchunks = cdiv(N, ENC_CHUNK);
  const int c4 = C / 4;
  const int threads = c4 <= 256 ? (c4 + 31) / 32 * 32 : 256;
  dim3 grid(nchunks, cdiv(c4, threads));
  enc_chunk_kernel<<<grid, threads, 0, st>>>(sorted_keys, dx0, dwte, chunk_part, N, C);
  enc_fixup_kernel<<<grid, threads, 0, st>>>(sorted_keys, dwte, chunk_part, N, C, nchunks);
  const int tc4 = T * c4;
  dwpe_kernel<<<grid_for(tc4, 256), 256, 0, st>>>(reinterpret_cast<const float4*>(dx0),
                                                  reinterpret_cast<float4*>(dwpe), B, tc4);
  note_kernel_launches(5);
  return ok();
}

int launch_topk_sample(cudaStream_t st, bool is_bf16, const void* logits, long long ld, int n_rows, const int* rows,
                       const float* u, int n, int V, int k, int* out, int* out_topk) {
  if (n <= 0 || n_rows <= 0 || V <= 0 || k <= 0 || k > TOPK_MAX || ld < V) return -4;
  if (k > V) k = V;
  if (is_bf16)
    topk_sample_kernel<bf16><<<n, TOPK_THREADS, 0, st>>>(static_cast<const bf16*>(logits), ld, n_rows, rows, u, V, k,
                                                         out, out_topk);
  else
    topk_sample_kernel<float><<<n, TOPK_THREADS, 0, st>>>(static_cast<const float*>(logits), ld, n_rows, rows, u, V,
                                                          k, out, out_topk);
  note_kernel_launches(1);
  return ok();
}

int launch_global_norm(cudaStream_t st, const float* g, long long n, double* part, int nparts, float clip,
                       float* out2) {
  sumsq_kernel<<<nparts, 512, 0, st>>>(g, n, part);
  norm_finalize_kernel<<<1, 256, 0, st>>>(part, nparts, clip, out2);
  note_kernel_launches(2);
  return ok();
}

int launch_adamw(cudaStream_t st, float* p, const float* g, float* m, float* v, uint16_t* shadow,
                 const AdamBlock* blocks, int nblocks, const float* clip_scale, float lr, float b1, float b2,
                 float eps, float wd, float bc1, float bc2) {
  adamw_kernel<<<nblocks, 256, 0, st>>>(p, g, m, v, reinterpret_cast<bf16*>(shadow), blocks, clip_scale, lr, b1, b2,
                                        eps, wd, bc1, bc2);
  note_kernel_launches(1);
  return ok();
}

int launch_init_normal(cudaStream_t st, float* p, long long n, uint64_t state, double std) {
  init_normal_kernel<<<grid_for(n, 256), 256, 0, st>>>(p, n, state, std);
  note_kernel_launches(1);
  return ok();
}
int launch_fill(cudaStream_t st, float* p, long long n, float value) {
  fill_kernel<<<grid_for(n, 256), 256, 0, st>>>(p, n, value);
  note_kernel_launches(1);
  return ok();
}
int launch_cast_bf16(cudaStream_t st, const float* src, uint16_t* dst, long long n) {
  cast_bf16_kernel<<<grid_for(n, 256), 256, 0, st>>>(src, reinterpret_cast<bf16*>(dst), n);
  note_kernel_launches(1);
  return ok();
}
