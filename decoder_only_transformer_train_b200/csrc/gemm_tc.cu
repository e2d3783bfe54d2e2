// bf16 x bf16 -> fp32 GEMM on the sm_100a tensor cores (tcgen05.mma, accumulators in
// TMEM), fed by TMA with a multi-stage mbarrier pipeline, with fused epilogues.
//
// Roles inside one persistent CTA (320 threads, one CTA per SM):
//   warp 0      : TMA producer (one elected lane) - stages of A and B tiles
//   warp 1      : TMEM allocator + MMA issuer (one elected lane)
//   warps 2..9  : epilogue - tcgen05.ld of the fp32 accumulator, fused math, stores;
//                 two warps per TMEM lane quarter, each taking half of the tile's columns
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue of one
// output tile overlaps the main loop of the next.
//
// The products are those of the pages' Linear layers (nn.Linear y = x W^T + b, "Karpathy's
// Zero to Hero, Lecture 9: Reproduce GPT-2 (124M)" notes, "Code you'll write") and of the
// tied lm_head; the epilogues fuse the bias, the residual add, the tanh-GELU and its
// derivative, and the softmax partials of the cross-entropy.
#include "sm100.cuh"
#include "gemm.h"
#include "kernels.h"

namespace {

constexpr int BM = 128;
constexpr int BK = 64;             // 64 bf16 = one 128-byte swizzle row
constexpr int NUM_THREADS = 320;
constexpr int EPI_THREADS = 256;

template <int BN>
struct TileCfg {
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 192 ? 5 : 6);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;   // +1024: manual alignment
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;   // power of two >= 2*BN
};

struct TileSched {
  int m_tiles, n_tiles, splits, nk, kb_per_split;
  __device__ __forceinline__ int num_tiles() const { return m_tiles * n_tiles * splits; }
  __device__ __forceinline__ void decode(int t, int& tm, int& tn, int& split, int& kb0, int& kb1) const {
    const int mn = m_tiles * n_tiles;
    split = t / mn;
    const int r = t - split * mn;
    tm = r % m_tiles;
    tn = r / m_tiles;
    kb0 = split * kb_per_split;
    kb1 = min(nk, kb0 + kb_per_split);
  }
};

__device__ __forceinline__ void load_f32x32(const float* p, float (&o)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 q = reinterpret_cast<const float4*>(p)[i];
    o[4 * i] = q.x; o[4 * i + 1] = q.y; o[4 * i + 2] = q.z; o[4 * i + 3] = q.w;
  }
}
__device__ __forceinline__ void store_f32x32(float* p, const float (&o)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}
__device__ __forceinline__ void store_bf16x32(bf16* p, const float (&o)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 q;
    q.x = pack_bf16x2(o[8 * i + 0], o[8 * i + 1]);
    q.y = pack_bf16x2(o[8 * i + 2], o[8 * i + 3]);
    q.z = pack_bf16x2(o[8 * i + 4], o[8 * i + 5]);
    q.w = pack_bf16x2(o[8 * i + 6], o[8 * i + 7]);
    reinterpret_cast<uint4*>(p)[i] = q;
  }
}
__device__ __forceinline__ void load_bf16x32(const bf16* p, float (&o)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 q = reinterpret_cast<const uint4*>(p)[i];
    float2 a = unpack_bf16x2(q.x), b = unpack_bf16x2(q.y), c = unpack_bf16x2(q.z), d = unpack_bf16x2(q.w);
    o[8 * i + 0] = a.x; o[8 * i + 1] = a.y; o[8 * i + 2] = b.x; o[8 * i + 3] = b.y;
    o[8 * i + 4] = c.x; o[8 * i + 5] = c.y; o[8 * i + 6] = d.x; o[8 * i + 7] = d.y;
  }
}

struct CeRowState {
  float mx, sum, amax;
  int aidx;
};

// Epilogue of one 32-column chunk of one output row.
__device__ __forceinline__ void epilogue_chunk(const EpiParams& ep, int m, int n0, float (&v)[32], int split,
                                               CeRowState& ce) {
  const int N = ep.N;
  const bool full = (n0 + 32 <= N);
  const int nvalid = full ? 32 : max(0, N - n0);
  const float alpha = ep.alpha;
  float b[32];
  if (ep.bias != nullptr && ep.kind != EPI_SPLITK && ep.kind != EPI_ACCUM_F32 && ep.kind != EPI_CE_FWD &&
      ep.kind != EPI_GELU_BWD) {
    if (full) {
      load_f32x32(ep.bias + n0, b);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) b[j] = (j < nvalid) ? ep.bias[n0 + j] : 0.0f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) b[j] = 0.0f;
  }

  switch (ep.kind) {
    case EPI_STORE_ACT: {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = alpha * v[j] + b[j];
      bf16* c = reinterpret_cast<bf16*>(ep.C) + (long long)m * ep.ldc + n0;
      if (full) store_bf16x32(c, v);
      else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) c[j] = __float2bfloat16_rn(v[j]);
      }
      break;
    }
    case EPI_STORE_F32: {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = alpha * v[j] + b[j];
      float* c = reinterpret_cast<float*>(ep.C) + (long long)m * ep.ldc + n0;
      if (full) store_f32x32(c, v);
      else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) c[j] = v[j];
      }
      break;
    }
    case EPI_ACCUM_F32: {
      float* c = reinterpret_cast<float*>(ep.C) + (long long)m * ep.ldc + n0;
      if (full) {
        float o[32];
        load_f32x32(c, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] += alpha * v[j];
        store_f32x32(c, o);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) c[j] += alpha * v[j];
      }
      break;
    }
    case EPI_RESID_F32: {
      const float* r = reinterpret_cast<const float*>(ep.aux) + (long long)m * ep.ld_aux + n0;
      float* c = reinterpret_cast<float*>(ep.C) + (long long)m * ep.ldc + n0;
      if (full) {
        float o[32];
        load_f32x32(r, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] += alpha * v[j] + b[j];
        store_f32x32(c, o);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) c[j] = r[j] + alpha * v[j] + b[j];
      }
      break;
    }
    case EPI_GELU_FWD: {
      bf16* u = reinterpret_cast<bf16*>(ep.aux_out) + (long long)m * ep.ld_aux_out + n0;
      bf16* c = reinterpret_cast<bf16*>(ep.C) + (long long)m * ep.ldc + n0;
      float g[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] = alpha * v[j] + b[j];
        g[j] = gelu_tanh_fast(v[j]);
      }
      if (full) {
        store_bf16x32(u, v);
        store_bf16x32(c, g);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) {
            u[j] = __float2bfloat16_rn(v[j]);
            c[j] = __float2bfloat16_rn(g[j]);
          }
      }
      break;
    }
    case EPI_GELU_BWD: {
      const bf16* u = reinterpret_cast<const bf16*>(ep.aux) + (long long)m * ep.ld_aux + n0;
      bf16* c = reinterpret_cast<bf16*>(ep.C) + (long long)m * ep.ldc + n0;
      if (full) {
        float uu[32];
        load_bf16x32(u, uu);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = alpha * v[j] * gelu_tanh_grad_fast(uu[j]);
        store_bf16x32(c, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) c[j] = __float2bfloat16_rn(alpha * v[j] * gelu_tanh_grad_fast(__bfloat162float(u[j])));
      }
      break;
    }
    case EPI_CE_FWD: {
      bf16* c = reinterpret_cast<bf16*>(ep.C) + (long long)m * ep.ldc + n0;
      float cmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] *= alpha;
        if (j < nvalid) {
          if (v[j] > ce.amax) { ce.amax = v[j]; ce.aidx = n0 + j; }
          cmax = fmaxf(cmax, v[j]);
        }
      }
      if (nvalid > 0) {
        const float nmx = fmaxf(ce.mx, cmax);
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) s += __expf(v[j] - nmx);
        ce.sum = ce.sum * __expf(ce.mx - nmx) + s;
        ce.mx = nmx;
        const int y = ep.targets[m];
        if (y >= n0 && y < n0 + nvalid) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (n0 + j == y) ep.zt[m] = v[j];
        }
      }
      if (full) store_bf16x32(c, v);
      else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) c[j] = __float2bfloat16_rn(v[j]);
      }
      break;
    }
    case EPI_SPLITK: {
      float* w = ep.ws + ((long long)split * ep.M + m) * (long long)N + n0;
      if (full && (N % 4 == 0)) store_f32x32(w, v);
      else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) w[j] = v[j];
      }
      break;
    }
    default:
      break;
  }
}

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               TileSched sched, EpiParams ep) {
  using Cfg = TileCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Cfg::STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty_bar = full_bar + Cfg::STAGES;
  uint64_t* tfull_bar = empty_bar + Cfg::STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], EPI_THREADS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = sched.num_tiles();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int tm, tn, split, kb0, kb1;
        sched.decode(t, tm, tn, split, kb0, kb1);
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sA = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* sB = sA + Cfg::A_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::STAGE_BYTES);
          const int k0 = kb * BK;
          if (!A_MN) {
            tma_load_2d(sA, &tmA, k0, m0, &full_bar[stage]);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j) tma_load_2d(sA + j * 8192, &tmA, m0 + 64 * j, k0, &full_bar[stage]);
          }
          if (!B_MN) {
            tma_load_2d(sB, &tmB, k0, n0, &full_bar[stage]);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(sB + j * 8192, &tmB, n0 + 64 * j, k0, &full_bar[stage]);
          }
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = make_idesc_bf16(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int tm, tn, split, kb0, kb1;
        sched.decode(t, tm, tn, split, kb0, kb1);
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t aBase = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t bBase = aBase + Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? make_sdesc_sw128(aBase + k * 2048, 8192, 1024)
                                     : make_sdesc_sw128(aBase + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? make_sdesc_sw128(bBase + k * 2048, 8192, 1024)
                                     : make_sdesc_sw128(bBase + k * 32, 16, 1024);
            tc_mma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty_bar[stage]);
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;        // which half of the tile's columns
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int tm, tn, split, kb0, kb1;
      sched.decode(t, tm, tn, split, kb0, kb1);
      if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const int m = tm * BM + row;
      const int n_base = tn * BN;
      CeRowState ce{-INFINITY, 0.0f, -INFINITY, 0x7fffffff};
#pragma unroll 1
      for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + acc * BN + c + (static_cast<uint32_t>(q * 32) << 16), r);
        tmem_wait_ld();
        if (m < ep.M && n_base + c < ep.N) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          epilogue_chunk(ep, m, n_base + c, v, split, ce);
        }
      }
      if (ep.kind == EPI_CE_FWD && m < ep.M) {
        CePartial p;
        p.max = ce.mx;
        p.sum = ce.sum;
        p.amax = ce.amax;
        p.aidx = ce.aidx;
        ep.ce_part[(long long)m * ep.n_ctiles + tn * 2 + half] = p;
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// split-K reduction in fixed split order: C[m,n] += alpha * sum_s ws[s][m][n]
__global__ void splitk_reduce_kernel(float* __restrict__ C, long long ldc, const float* __restrict__ ws, int M,
                                     int N, int splits, float alpha) {
  const long long total = (long long)M * N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i / N), n = (int)(i % N);
    float s = 0.0f;
    for (int k = 0; k < splits; ++k) s += ws[(long long)k * total + i];
    C[(long long)m * ldc + n] += alpha * s;
  }
}

typedef CUresult (*PFN_tmapEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                         const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                         CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                         CUtensorMapFloatOOBfill);

PFN_tmapEncodeTiled get_encode_fn() {
  static PFN_tmapEncodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_tmapEncodeTiled>(p);
  }
  return fn;
}

// bf16 2-D tensor map: `inner` contiguous elements per row, `outer` rows, row pitch ld.
int encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                   uint32_t box_inner, uint32_t box_outer) {
  PFN_tmapEncodeTiled fn = get_encode_fn();
  if (fn == nullptr) return -3;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (ld * 2) % 16 != 0) return -1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -3;
}

template <int BN, bool A_MN, bool B_MN>
int launch_tc(cudaStream_t st, const CUtensorMap& ta, const CUtensorMap& tb, TileSched sched, const EpiParams& ep,
              int num_sms) {
  using Cfg = TileCfg<BN>;
  auto kern = gemm_tc_kernel<BN, A_MN, B_MN>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) != cudaSuccess)
      return -3;
    attr_set = true;
  }
  const int tiles = sched.m_tiles * sched.n_tiles * sched.splits;
  const int grid = tiles < num_sms ? tiles : num_sms;
  kern<<<grid, NUM_THREADS, Cfg::SMEM, st>>>(ta, tb, sched, ep);
  note_kernel_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace

int gemm_tc_tile_n(int N) { return N > 128 ? 256 : 128; }
int gemm_tc_ce_tiles(int N) { return cdiv(N, gemm_tc_tile_n(N)) * 2; }

namespace {
// Picks the output tile width (128, 192 or 256 columns) and the number of K splits from a
// small cost model in MMA clock cycles: the busiest SM's tiles x the tile's main loop
// (narrower tiles re-read more operand bytes per FLOP, hence the efficiency factor), plus
// for split-K the extra fp32 traffic of the partials and their reduction.
struct TileChoice {
  int bn, splits;
};
TileChoice choose_tiles(int M, int N, int K, bool can_split, size_t ws_elems, int num_sms, bool fixed_bn) {
  const int m_tiles = cdiv(M, BM);
  const int nk = cdiv(K, BK);
  const int bns[3] = {256, 192, 128};
  const double eff[3] = {1.0, 0.96, 0.88};
  TileChoice best{gemm_tc_tile_n(N), 1};
  double best_cost = 1e300;
  for (int i = 0; i < 3; ++i) {
    const int bn = bns[i];
    if (fixed_bn && bn != gemm_tc_tile_n(N)) continue;
    if (bn > 128 && N <= 128) continue;
    const int tiles = m_tiles * cdiv(N, bn);
    for (int sp = 1; sp <= (can_split ? 8 : 1); ++sp) {
      if (sp > 1 && (nk / sp < 8 || (size_t)sp * M * N > ws_elems)) break;
      const int kb = cdiv(nk, sp);
      const double per_tile = (double)bn * kb * 2.0 / eff[i] + 1500.0;   // MMA clks of a 128 x bn x 64kb tile + overhead
      const double waves = (double)cdiv(tiles * sp, num_sms);
      double cost = waves * per_tile;
      if (sp > 1) cost += (double)(sp + 2) * M * N * 4.0 / 6.0e12 * 1.9e9 + 3000.0;   // partial traffic + reduce launch
      if (cost < best_cost * 0.999) {
        best_cost = cost;
        best = TileChoice{bn, sp};
      }
    }
  }
  return best;
}
}  // namespace

int gemm_bf16_tc(cudaStream_t st, int M, int N, int K, const void* A, long long lda, bool a_mn, const void* B,
                 long long ldb, bool b_mn, EpiParams ep, float* ws, size_t ws_elems, int num_sms) {
  if (M <= 0 || N <= 0) return 0;
  if (K <= 0) return -1;
  if (a_mn && !b_mn) return -1;   // not needed by any Linear-layer product
  ep.M = M;
  ep.N = N;
  // alignment of the vectorised epilogue accesses
  if (ep.kind != EPI_SPLITK && (ep.ldc % 8) != 0) return -1;
  const bool can_split = (ep.kind == EPI_ACCUM_F32 && ws != nullptr);
  // the softmax partials of EPI_CE_FWD are laid out per 256/128-column tile
  const TileChoice tc = choose_tiles(M, N, K, can_split, ws_elems, num_sms, ep.kind == EPI_CE_FWD);
  const int BN = tc.bn;
  CUtensorMap ta, tb;
  int rc;
  if (!a_mn) rc = encode_bf16_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda, BK, BM);
  else rc = encode_bf16_2d(&ta, A, (uint64_t)M, (uint64_t)K, (uint64_t)lda, 64, BK);
  if (rc) return rc;
  if (!b_mn) rc = encode_bf16_2d(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)ldb, BK, (uint32_t)BN);
  else rc = encode_bf16_2d(&tb, B, (uint64_t)N, (uint64_t)K, (uint64_t)ldb, 64, BK);
  if (rc) return rc;

  TileSched sched;
  sched.m_tiles = cdiv(M, BM);
  sched.n_tiles = cdiv(N, BN);
  sched.nk = cdiv(K, BK);
  sched.splits = 1;
  sched.kb_per_split = sched.nk;
  EpiParams run = ep;
  bool split = false;
  if (tc.splits > 1) {
    sched.kb_per_split = cdiv(sched.nk, tc.splits);
    sched.splits = cdiv(sched.nk, sched.kb_per_split);
    run.kind = EPI_SPLITK;
    run.ws = ws;
    split = true;
  }
  if (ep.kind == EPI_CE_FWD) {
    run.n_ctiles = sched.n_tiles * 2;
    run.ce_tile_n = BN / 2;
  }
#define LAUNCH_BN(BNV)                                                                           \
  do {                                                                                           \
    if (!a_mn && !b_mn) rc = launch_tc<BNV, false, false>(st, ta, tb, sched, run, num_sms);     \
    else if (!a_mn && b_mn) rc = launch_tc<BNV, false, true>(st, ta, tb, sched, run, num_sms);  \
    else rc = launch_tc<BNV, true, true>(st, ta, tb, sched, run, num_sms);                       \
  } while (0)
  if (BN == 256) LAUNCH_BN(256);
  else if (BN == 192) LAUNCH_BN(192);
  else LAUNCH_BN(128);
#undef LAUNCH_BN
  if (rc) return rc;
  if (split) {
    const long long total = (long long)M * N;
    const int threads = 256;
    long long nb = cdivll(total, threads);
    if (nb > (long long)num_sms * 8) nb = (long long)num_sms * 8;
    const int blocks = (int)nb;
    splitk_reduce_kernel<<<blocks, threads, 0, st>>>(reinterpret_cast<float*>(ep.C), ep.ldc, ws, M, N,
                                                     sched.splits, ep.alpha);
    note_kernel_launches(1);
    if (cudaGetLastError() != cudaSuccess) return -3;
  }
  return 0;
}
