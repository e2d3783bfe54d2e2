// bf16 x bf16 -> fp32 GEMM on the sm_100a tensor cores (tcgen05.mma, accumulators in
// TMEM), fed by TMA with a multi-stage mbarrier pipeline, with fused epilogues.
//
// Roles inside one persistent CTA (320 threads, one CTA per SM):
//   warp 0      : TMA producer (one elected lane) - stages of A and B tiles
//   warp 1      : TMEM allocator + MMA issuer (one elected lane)
//   warps 2..9  : epilogue - tcgen05.ld of the fp32 accumulator, fused math; two warps
//                 per TMEM lane quarter, each taking half of the tile's columns.  Each warp
//                 owns a 32-row slab: thread r computes row r, writes it into a small
//                 64-byte-swizzled shared buffer, and one lane moves the 32 x 64-byte box
//                 to global memory with a TMA store (inputs the epilogue needs - residual,
//                 accumulator, GELU pre-activation - arrive the same way by TMA load), so
//                 global traffic is in full lines rather than per-row 16-byte pieces.
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue of one
// output tile overlaps the main loop of the next.
//
// The products are those of the pages' Linear layers (nn.Linear y = x W^T + b, "Karpathy's
// Zero to Hero, Lecture 9: Reproduce GPT-2 (124M)" notes, "Code you'll write") and of the
// tied lm_head; the epilogues fuse the bias, the residual add, the tanh-GELU and its
// derivative, and the softmax partials of the cross-entropy.
#include <stdlib.h>
#include "sm100.cuh"
#include "gemm.h"
#include "kernels.h"

namespace {

constexpr int BM = 128;
constexpr int BK = 64;             // 64 bf16 = one 128-byte swizzle row
constexpr int NUM_THREADS = 320;

constexpr int BOX_BYTES = 2048;     // one epilogue staging box: 32 rows x 64 bytes

// CG = 1: one CTA computes a 128 x BN tile.  CG = 2: a CTA pair (cluster of 2, tcgen05
// cta_group::2) computes a 256 x BN tile; each CTA stages its own 128 rows of A and
// BN / 2 rows of B, so a stage is smaller and the pipeline deeper.
// WIDE: single CTAs of the residual-add epilogue trade a main-loop stage for a ring of 4
// boxes, so more residual boxes load ahead (measured: 37.4 -> 35.5 us for the 768-column
// attention projection; the GELU epilogues lost more from the stage than they gained).
template <int BN, int CG = 1, bool WIDE = false>
struct TileCfg {
  static constexpr int B_ROWS = BN / CG;                      // rows of B staged by one CTA
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr bool WIDE_RING = WIDE && CG == 1 && BN >= 192;
  static constexpr int STAGES = CG == 1 ? (BN == 256 ? (WIDE_RING ? 3 : 4) : (BN == 192 ? 4 : 6))
                                        : (BN == 256 ? 5 : (BN == 192 ? 5 : 6));
  // epilogue staging boxes per warp: a pair's smaller stages leave room for a ring of 4, so
  // epilogue inputs can be loaded ahead
  static constexpr int NBOX = (CG == 2 || WIDE_RING) ? 4 : 2;
  static constexpr int STG_BYTES = 8 * NBOX * BOX_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG_BYTES + BAR_BYTES + 1024;   // +1024: manual alignment
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;   // power of two >= 2*BN
  static_assert((2 * STAGES + 4 + 8 * NBOX) * 8 + 8 <= BAR_BYTES, "GEMM barriers");
  static_assert(SMEM <= 232448, "GEMM shared memory");
  static_assert(CG == 1 || (BN / 2) % 16 == 0, "CTA-pair tile width");
};

// Tile order: with few column tiles (n_fast) the column tiles of one row block are
// neighbours, so the CTAs working on them at the same time share each A tile (read once
// from HBM); otherwise the row tiles of one column block are neighbours and share B.
struct TileSched {
  int m_tiles, n_tiles, splits, nk, kb_per_split, n_fast;
  __device__ __forceinline__ int num_tiles() const { return m_tiles * n_tiles * splits; }
  __device__ __forceinline__ void decode(int t, int& tm, int& tn, int& split, int& kb0, int& kb1) const {
    const int mn = m_tiles * n_tiles;
    split = t / mn;
    const int r = t - split * mn;
    if (n_fast) {
      tn = r % n_tiles;
      tm = r / n_tiles;
    } else {
      tm = r % m_tiles;
      tn = r / m_tiles;
    }
    kb0 = split * kb_per_split;
    kb1 = min(nk, kb0 + kb_per_split);
  }
};

struct CeRowState {
  float mx, sum, amax, zt;
  int aidx;
};

constexpr float CE_LOG2E = 1.4426950408889634f;

// Softmax partials of the cross-entropy for one 32-column chunk of one logits row, from
// the fp32 accumulator: running max and sum of exp(v - max) (online rescaling), the first
// column reaching the running maximum (argmax), and the target column's logit.  Columns
// at or past N (nvalid < 32) count as -inf.
__device__ __forceinline__ void ce_row_chunk(int n0, int nvalid, int y, const float (&v)[32], CeRowState& ce) {
  float w[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) w[j] = (j < nvalid) ? v[j] : -INFINITY;
  // chunk max as a shallow tree of 3-input maxima
  float t[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) t[i] = max3f(w[3 * i], w[3 * i + 1], w[3 * i + 2]);
  t[10] = fmaxf(w[30], w[31]);
  const float cmax = fmaxf(max3f(max3f(t[0], t[1], t[2]), max3f(t[3], t[4], t[5]), max3f(t[6], t[7], t[8])),
                           fmaxf(t[9], t[10]));
  if (cmax > ce.amax) {   // strictly greater: an earlier column keeps a tie
    uint32_t mask = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) mask |= (w[j] == cmax ? 1u : 0u) << j;
    ce.amax = cmax;
    ce.aidx = n0 + __ffs(mask) - 1;
  }
  const float nmx = fmaxf(ce.mx, cmax);
  const float2 l2e = make_float2(CE_LOG2E, CE_LOG2E);
  const float2 off = make_float2(-nmx * CE_LOG2E, -nmx * CE_LOG2E);
  float2 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 x = ffma2(make_float2(w[j], w[j + 1]), l2e, off);   // (v - max) log2 e
    acc[(j >> 1) & 3] = fadd2(acc[(j >> 1) & 3], make_float2(ex2(x.x), ex2(x.y)));
  }
  const float2 s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  ce.sum = ce.sum * ex2((ce.mx - nmx) * CE_LOG2E) + (s2.x + s2.y);
  ce.mx = nmx;
  const int jt = y - n0;
  if (jt >= 0 && jt < nvalid) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == jt) ce.zt = v[j];
  }
}

// Byte offset of 16-byte granule g (0..3) of row r in a 32 x 64-byte box stored with the
// TMA 64-byte swizzle (granule index XOR bits 7-8 of the address).
__device__ __forceinline__ uint32_t box_off(int r, int g) { return r * 64 + ((g ^ ((r >> 1) & 3)) << 4); }

__device__ __forceinline__ void box_put_bf16(uint8_t* box, int r, const float* v) {   // 32 values
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * g + 0], v[8 * g + 1]);
    w.y = pack_bf16x2(v[8 * g + 2], v[8 * g + 3]);
    w.z = pack_bf16x2(v[8 * g + 4], v[8 * g + 5]);
    w.w = pack_bf16x2(v[8 * g + 6], v[8 * g + 7]);
    *reinterpret_cast<uint4*>(box + box_off(r, g)) = w;
  }
}
__device__ __forceinline__ void box_get_bf16(const uint8_t* box, int r, float* v) {   // 32 values
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint4 w = *reinterpret_cast<const uint4*>(box + box_off(r, g));
    const float2 a = unpack_bf16x2(w.x), b = unpack_bf16x2(w.y), c = unpack_bf16x2(w.z), d = unpack_bf16x2(w.w);
    v[8 * g + 0] = a.x; v[8 * g + 1] = a.y; v[8 * g + 2] = b.x; v[8 * g + 3] = b.y;
    v[8 * g + 4] = c.x; v[8 * g + 5] = c.y; v[8 * g + 6] = d.x; v[8 * g + 7] = d.y;
  }
}
__device__ __forceinline__ void box_put_f32(uint8_t* box, int r, const float* v) {    // 16 values
#pragma unroll
  for (int g = 0; g < 4; ++g)
    *reinterpret_cast<float4*>(box + box_off(r, g)) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
}
__device__ __forceinline__ void box_get_f32(const uint8_t* box, int r, float* v) {    // 16 values
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float4 w = *reinterpret_cast<const float4*>(box + box_off(r, g));
    v[4 * g] = w.x; v[4 * g + 1] = w.y; v[4 * g + 2] = w.z; v[4 * g + 3] = w.w;
  }
}

// Epilogue classes, one kernel instantiation each, so that a kernel carries only its own
// epilogue code (the fused ones compile to straight-line code for their kind; the plain
// class is the bf16 store with bias, the fp32 class covers fp32 stores, fp32 accumulation
// and split-K partials at run time).
enum EpiClass : int { EK_PLAIN = 0, EK_RESID = 1, EK_GELU_FWD = 2, EK_GELU_BWD = 3, EK_CE = 4, EK_F32 = 5 };
inline int epi_class(int kind) {
  return kind == EPI_RESID_F32 ? EK_RESID
         : kind == EPI_GELU_FWD ? EK_GELU_FWD
         : kind == EPI_GELU_BWD ? EK_GELU_BWD
         : kind == EPI_CE_FWD   ? EK_CE
         : kind == EPI_STORE_ACT ? EK_PLAIN
                                 : EK_F32;
}

__device__ __forceinline__ bool kind_has_bias(int kind) {
  return kind == EPI_STORE_ACT || kind == EPI_STORE_F32 || kind == EPI_RESID_F32 || kind == EPI_GELU_FWD;
}
__device__ __forceinline__ bool kind_out_bf16(int kind) {
  return kind == EPI_STORE_ACT || kind == EPI_GELU_FWD || kind == EPI_GELU_BWD || kind == EPI_CE_FWD;
}

// Per-warp epilogue state: a ring of NB staging boxes, each with an mbarrier for TMA loads of
// epilogue inputs.  Boxes are handed out in ring order and every box handed out ends in
// exactly one TMA store (one bulk group), so allocation a is store group a: before
// allocation a reuses its box, the store of allocation a - NB must have read it.
template <int NB>
struct EpiRing {
  uint8_t* boxes;
  uint64_t* bars;
  uint32_t phases;          // bit i: parity of the next completion of bars[i]
  uint32_t inflight;        // bit i: a load into box i not yet waited for
  int alloc;                // boxes handed out so far
  int stores;               // store groups committed so far
  volatile int* abort_flag;
  int lane;
  __device__ __forceinline__ uint8_t* box(int i) const { return boxes + i * BOX_BYTES; }
  __device__ __forceinline__ int take() {
    const int a = alloc++;
    const int pend = stores - 1 - (a - NB);   // store groups that may stay in flight
    if (a >= NB && lane == 0) {
      if (pend <= 0) bulk_wait_group_read<0>();
      else if (pend == 1 || NB == 2) bulk_wait_group_read<1>();
      else if (pend == 2) bulk_wait_group_read<2>();
      else bulk_wait_group_read<3>();
    }
    __syncwarp();
    return a % NB;
  }
  __device__ __forceinline__ void issue_load(int i, const CUtensorMap* map, int x, int y) {
    inflight |= 1u << i;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[i], BOX_BYTES);
      tma_load_2d(box(i), map, x, y, &bars[i]);
    }
  }
  // the whole warp waits (warp-uniform outcome)
  __device__ __forceinline__ bool wait_load(int i) {
    const bool ok = mbar_wait_warp(&bars[i], (phases >> i) & 1u, abort_flag);
    if (ok) {
      phases ^= 1u << i;
      inflight &= ~(1u << i);
    }
    return ok;
  }
  // after an abort: lets the loads still in flight land before the CTA leaves
  __device__ __forceinline__ void drain() {
    if (lane == 0)
      for (int i = 0; i < NB; ++i)
        if ((inflight >> i) & 1u) mbar_drain(&bars[i], (phases >> i) & 1u);
    __syncwarp();
  }
  __device__ __forceinline__ void store(int i, const CUtensorMap* map, int x, int y) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(map, x, y, box(i));
      bulk_commit_group();
    }
    ++stores;
  }
};

template <int BN, bool A_MN, bool B_MN, int CG, int EK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmIn,
               const __grid_constant__ CUtensorMap tmOut2, TileSched sched, EpiParams ep) {
  using Cfg = TileCfg<BN, CG, EK == EK_RESID>;
  constexpr int BMT = BM * CG;                       // rows of an output tile
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;   // 0: the pair's leader (issues the MMAs)
  const int cl_id = blockIdx.x / CG, n_cl = gridDim.x / CG;   // tiles are dealt per CTA group
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stg = smem + Cfg::STAGES * Cfg::STAGE_BYTES;                       // epilogue boxes
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(stg + Cfg::STG_BYTES);
  uint64_t* empty_bar = full_bar + Cfg::STAGES;
  uint64_t* tfull_bar = empty_bar + Cfg::STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* epi_bar = tempty_bar + 2;             // [8][NBOX] per epilogue warp and box
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + 8 * Cfg::NBOX);
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
      mbar_init(&tempty_bar[a], 8 * CG);   // one arrival per epilogue warp of every CTA of the group
    }
    for (int w = 0; w < 8 * Cfg::NBOX; ++w) mbar_init(&epi_bar[w], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
    tma_prefetch_desc(&tmIn);
    tma_prefetch_desc(&tmOut2);
  }
  if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (CG == 2) cluster_sync();   // the peer's barriers are initialised before any cross-CTA signal
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = sched.num_tiles();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;            // stages filled so far
      bool ok = true;
      // this CTA's rows of A and of B within a tile; with a CTA pair both halves complete
      // on the leader's full barrier, which the leader arms for the bytes of both
      auto load = [&](void* dst, const CUtensorMap* map, int x, int y, int st) {
        if (CG == 2) tma_load_2d_pair(dst, map, x, y, cluster_addr(&full_bar[st], 0));
        else tma_load_2d(dst, map, x, y, &full_bar[st]);
      };
      for (int t = cl_id; t < ntiles && ok; t += n_cl) {
        int tm, tn, split, kb0, kb1;
        sched.decode(t, tm, tn, split, kb0, kb1);
        const int m0 = tm * BMT + (int)rank * BM, n0 = tn * BN + (int)rank * Cfg::B_ROWS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sA = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* sB = sA + Cfg::A_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], CG * Cfg::STAGE_BYTES);
          const int k0 = kb * BK;
          if (!A_MN) {
            load(sA, &tmA, k0, m0, stage);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j) load(sA + j * 8192, &tmA, m0 + 64 * j, k0, stage);
          }
          if (!B_MN) {
            load(sB, &tmB, k0, n0, stage);
          } else {
#pragma unroll
            for (int j = 0; j < Cfg::B_ROWS / 64; ++j) load(sB + j * 8192, &tmB, n0 + 64 * j, k0, stage);
          }
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1; }
          ++issued;
        }
      }
      // after an abort, the loads still in flight land before the CTA leaves (the leader's
      // full barriers count the bytes of both CTAs of a pair)
      if (*abort_flag && rank == 0)
        for (int s = 0; s < Cfg::STAGES && s < issued; ++s) {
          const int fills = (issued - 1 - s) / Cfg::STAGES + 1;
          mbar_drain(&full_bar[s], (uint32_t)((fills - 1) & 1));
        }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------------------ MMA issuer (the leader)
      // the whole warp runs the loop (descriptors and counters stay warp-uniform); one elected
      // lane issues the MMAs and commits
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc = make_idesc_bf16(BMT, BN, A_MN, B_MN);
      // operand descriptors of stage 0; each MMA's is derived by an add
      const uint64_t dA0 = A_MN ? make_sdesc_sw128(smem_u32(smem), 8192, 1024) : make_sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t dB0 = B_MN ? make_sdesc_sw128(smem_u32(smem) + Cfg::A_BYTES, 8192, 1024)
                                : make_sdesc_sw128(smem_u32(smem) + Cfg::A_BYTES, 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = cl_id; t < ntiles && ok; t += n_cl) {
        int tm, tn, split, kb0, kb1;
        sched.decode(t, tm, tn, split, kb0, kb1);
        const bool got = (CG == 2) ? mbar_wait_cluster(&tempty_bar[acc], acc_phase ^ 1, abort_flag)
                                   : mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_warp(&full_bar[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t aBase = sdesc_add(dA0, stage * Cfg::STAGE_BYTES);
          const uint64_t bBase = sdesc_add(dB0, stage * Cfg::STAGE_BYTES);
          if (leader) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint64_t ad = sdesc_add(aBase, A_MN ? k * 2048 : k * 32);
              const uint64_t bd = sdesc_add(bBase, B_MN ? k * 2048 : k * 32);
              if (CG == 2) tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
              else tc_mma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            }
            if (CG == 2) tc_commit_pair(&empty_bar[stage], 0x3);   // both CTAs' stage is free
            else tc_commit(&empty_bar[stage]);
          }
          __syncwarp();
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (leader) {
          if (CG == 2) tc_commit_pair(&tfull_bar[acc], 0x3);     // both halves of D are ready
          else tc_commit(&tfull_bar[acc]);
        }
        __syncwarp();
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    constexpr int NB = Cfg::NBOX;
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;        // which half of the tile's columns
    const int row = q * 32 + lane;
    const int ew = warp - 2;
    EpiRing<NB> E;
    E.boxes = stg + ew * NB * BOX_BYTES;
    E.bars = &epi_bar[ew * NB];
    E.phases = 0;
    E.inflight = 0;
    E.alloc = 0;
    E.stores = 0;
    E.abort_flag = abort_flag;
    E.lane = lane;
    // the fused classes fix their kind at compile time
    const int kind = (EK == EK_RESID)      ? (int)EPI_RESID_F32
                     : (EK == EK_GELU_FWD) ? (int)EPI_GELU_FWD
                     : (EK == EK_GELU_BWD) ? (int)EPI_GELU_BWD
                     : (EK == EK_CE)       ? (int)EPI_CE_FWD
                     : (EK == EK_PLAIN)    ? (int)EPI_STORE_ACT
                                           : ep.kind;
    const bool out_bf16 = (EK != EK_F32) && kind_out_bf16(kind);
    const bool use_bias = ep.bias != nullptr && kind_has_bias(kind);
    const float alpha = ep.alpha;
    // inputs read into the staging boxes and overwritten there by the result: residual or
    // accumulator (fp32, two 16-column boxes per 32-column chunk) or the GELU pre-activation
    // (bf16, one box per chunk).  The first NB boxes of them are requested before the
    // accumulator is ready; later ones as boxes retire.
    const bool has_in = (EK == EK_RESID || kind == EPI_ACCUM_F32 || EK == EK_GELU_BWD);
    const CUtensorMap* in_map = (kind == EPI_ACCUM_F32) ? &tmOut : &tmIn;
    const int depth = out_bf16 ? NB : NB / 2;   // chunks loaded ahead
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    // the leader's TMEM-empty barrier: every epilogue warp of the CTA group arrives once per tile
    const uint32_t tempty_leader0 = (CG == 2) ? cluster_addr(&tempty_bar[0], 0) : 0u;
    for (int t = cl_id; t < ntiles && ok; t += n_cl) {
      int tm, tn, split, kb0, kb1;
      sched.decode(t, tm, tn, split, kb0, kb1);
      const int row0 = tm * BMT + (int)rank * BM;               // this CTA's rows of the tile
      const int m = row0 + row;
      const int m_warp = row0 + q * 32;                         // first row of this warp's slab
      const int y_out = (kind == EPI_SPLITK) ? split * ep.ld_aux + m_warp : m_warp;   // ws rows per split: ld_aux
      const int c_begin = tn * BN + half * (BN / 2);            // first column of this warp's half tile
      // 32-column chunks of the half tile that start inside the matrix (warp-uniform)
      int nch = 0;
      if (m_warp < ep.M && c_begin < ep.N) nch = min(BN / 64, (ep.N - c_begin + 31) / 32);
      // fp32 boxes of chunk c: two, or one when its second 16 columns lie past N
      auto nbox_of = [&](int c) -> int { return out_bf16 ? 1 : ((c_begin + 32 * c + 16 < ep.N) ? 2 : 1); };
      auto load_chunk = [&](int c) {
        const int nb = nbox_of(c);
        for (int i = 0; i < nb; ++i) {
          const int bi = E.take();
          E.issue_load(bi, in_map, c_begin + 32 * c + 16 * i, m_warp);
        }
      };
      const int in_first = E.alloc;                             // allocation index of chunk 0's first input box
      if (has_in)
        for (int c = 0; c < min(depth, nch); ++c) load_chunk(c);
      CeRowState ce{-INFINITY, 0.0f, -INFINITY, 0.0f, 0x7fffffff};
      const int y_row = (EK == EK_CE && m < ep.M) ? ep.targets[m] : -1;
      if (!mbar_wait_warp(&tfull_bar[acc], acc_phase, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < nch && ok; ++c) {
        const int col = half * (BN / 2) + 32 * c;               // column within the tile
        const int n0 = c_begin + 32 * c;
        uint32_t r[32];
        tmem_ld32(tmem_base + acc * BN + col + (static_cast<uint32_t>(q * 32) << 16), r);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (EK == EK_CE && m < ep.M) ce_row_chunk(n0, min(32, ep.N - n0), y_row, v, ce);
        if (out_bf16) {
          float b[32];
          if (use_bias && n0 + 32 <= ep.N) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 q4 = reinterpret_cast<const float4*>(ep.bias + n0)[i];
              b[4 * i] = q4.x; b[4 * i + 1] = q4.y; b[4 * i + 2] = q4.z; b[4 * i + 3] = q4.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) b[j] = (use_bias && n0 + j < ep.N) ? ep.bias[n0 + j] : 0.f;
          }
          if (EK == EK_GELU_FWD) {
            // gelu(u) and gelu'(u) from one tanh, in pairs; gelu'(u) is what the backward needs
            float gp[32], g[32];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float2 gl, gd;
              gelu2_and_grad_fast(ffma2(make_float2(alpha, alpha), make_float2(v[j], v[j + 1]), make_float2(b[j], b[j + 1])),
                                  gl, gd);
              g[j] = gl.x; g[j + 1] = gl.y;
              gp[j] = gd.x; gp[j + 1] = gd.y;
            }
            int bx = E.take();
            box_put_bf16(E.box(bx), lane, gp);
            E.store(bx, &tmOut2, n0, m_warp);
            bx = E.take();
            box_put_bf16(E.box(bx), lane, g);
            E.store(bx, &tmOut, n0, m_warp);
          } else if (EK == EK_GELU_BWD) {
            const int bx = (in_first + c) % NB;
            if (!E.wait_load(bx)) { ok = false; break; }
            float u[32];
            box_get_bf16(E.box(bx), lane, u);
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 o = fmul2(fmul2(make_float2(alpha, alpha), make_float2(v[j], v[j + 1])),
                                     make_float2(u[j], u[j + 1]));
              u[j] = o.x;
              u[j + 1] = o.y;
            }
            box_put_bf16(E.box(bx), lane, u);
            E.store(bx, &tmOut, n0, m_warp);
            if (ep.colsum_part != nullptr) {
              // the warp's 32 rows summed per column (rows past M left out), 16 columns per pass
              float* prow = ep.colsum_part + (long long)(m_warp >> 5) * ep.N;
#pragma unroll
              for (int h16 = 0; h16 < 2; ++h16) {
                float x[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) x[j] = (m < ep.M) ? u[16 * h16 + j] : 0.f;
                const float cs = warp_colsum16(x, lane);
                const int n = n0 + 16 * h16 + (lane >> 1);
                if ((lane & 1) == 0 && n < ep.N) prow[n] = cs;
              }
            }
            if (c + depth < nch) load_chunk(c + depth);
          } else {   // EPI_STORE_ACT, EPI_CE_FWD
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 o = ffma2(make_float2(alpha, alpha), make_float2(v[j], v[j + 1]), make_float2(b[j], b[j + 1]));
              v[j] = o.x;
              v[j + 1] = o.y;
            }
            const int bx = E.take();
            box_put_bf16(E.box(bx), lane, v);
            E.store(bx, &tmOut, n0, m_warp);
          }
        } else {
          // fp32 output: two 16-column boxes
          const int ib = in_first + 2 * c;                      // allocation index of chunk c's first input box
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int n1 = n0 + hh * 16;
            if (!ok || n1 >= ep.N) continue;
            float o[16];
            if (kind == EPI_SPLITK) {
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] = v[hh * 16 + j];
            } else {
              float bj[16];
              if (use_bias && n1 + 16 <= ep.N) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float4 q4 = reinterpret_cast<const float4*>(ep.bias + n1)[i];
                  bj[4 * i] = q4.x; bj[4 * i + 1] = q4.y; bj[4 * i + 2] = q4.z; bj[4 * i + 3] = q4.w;
                }
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) bj[j] = (use_bias && n1 + j < ep.N) ? ep.bias[n1 + j] : 0.f;
              }
#pragma unroll
              for (int j = 0; j < 16; j += 2) {
                const float2 r2 = ffma2(make_float2(alpha, alpha), make_float2(v[hh * 16 + j], v[hh * 16 + j + 1]),
                                        make_float2(bj[j], bj[j + 1]));
                o[j] = r2.x;
                o[j + 1] = r2.y;
              }
            }
            int bx;
            if (has_in) {
              bx = (ib + hh) % NB;
              if (!E.wait_load(bx)) { ok = false; continue; }
              float in[16];
              box_get_f32(E.box(bx), lane, in);
              __syncwarp();
#pragma unroll
              for (int j = 0; j < 16; j += 2) {
                const float2 r2 = fadd2(make_float2(o[j], o[j + 1]), make_float2(in[j], in[j + 1]));
                o[j] = r2.x;
                o[j + 1] = r2.y;
              }
            } else {
              bx = E.take();
            }
            box_put_f32(E.box(bx), lane, o);
            E.store(bx, &tmOut, n1, y_out);
          }
          if (ok && has_in && c + depth < nch) load_chunk(c + depth);
        }
      }
      if (EK == EK_CE && m < ep.M) {
        CePartial p;
        p.max = ce.mx;
        p.sum = ce.sum;
        p.amax = ce.amax;
        p.aidx = ce.aidx;
        ep.ce_part[(long long)m * ep.n_ctiles + tn * 2 + half] = p;
        if (y_row >= c_begin && y_row < min(c_begin + BN / 2, ep.N)) ep.zt[m] = ce.zt;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2) mbar_arrive_cluster(tempty_leader0 + acc * 8);
        else mbar_arrive(&tempty_bar[acc]);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (!ok) E.drain();
    if (lane == 0) bulk_wait_group<0>();      // every store of this warp has landed
    __syncwarp();
  }

  tc_fence_before();
  if (CG == 2) cluster_sync();   // neither CTA leaves while its peer may still signal it
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (CG == 2) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    else tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// split-K reduction in fixed split order: C[m,n] += alpha * sum_s ws[s][m][n]
// ws holds `splits` (<= 8) partial products of Mpad rows each (row-major, N columns).  Each
// thread handles 4 consecutive columns with 16-byte accesses (N % 4 == 0, ldc % 4 == 0 and a
// 16-byte aligned C, which the fp32 tensor maps of the split path already require) and has
// all the splits' loads in flight before it adds them in split order.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(float* __restrict__ C, long long ldc,
                                                            const float* __restrict__ ws, int M, int Mpad, int N,
                                                            int splits, float alpha) {
  const int nq = N >> 2;
  const long long total = (long long)M * nq;
  const long long per_split = (long long)Mpad * N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i / nq), q = (int)(i - (long long)m * nq);
    const float* src = ws + (long long)m * N + 4 * q;
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < splits) v[k] = __ldcs(reinterpret_cast<const float4*>(src + k * per_split));
    float4 acc = v[0];
#pragma unroll
    for (int k = 1; k < 8; ++k)
      if (k < splits) {
        acc.x += v[k].x;
        acc.y += v[k].y;
        acc.z += v[k].z;
        acc.w += v[k].w;
      }
    float4* dst = reinterpret_cast<float4*>(C + (long long)m * ldc + 4 * q);
    float4 c = *dst;
    c.x += alpha * acc.x;
    c.y += alpha * acc.y;
    c.z += alpha * acc.z;
    c.w += alpha * acc.w;
    *dst = c;
  }
}

// The same with two consecutive float4 per thread (N % 8 == 0), every load of both issued
// before the adds, and one thread per pair: for the two-way splits of the weight gradients
// that is six 16-byte loads in flight per thread and a single pass over the grid.
__global__ void __launch_bounds__(256) splitk_reduce8_kernel(float* __restrict__ C, long long ldc,
                                                             const float* __restrict__ ws, int M, int Mpad, int N,
                                                             int splits, float alpha) {
  const int n8 = N >> 3;
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)M * n8) return;
  const long long per_split = (long long)Mpad * N;
  const int m = (int)(i / n8), q = (int)(i - (long long)m * n8);
  const float* src = ws + (long long)m * N + 8 * q;
  float4* dst = reinterpret_cast<float4*>(C + (long long)m * ldc + 8 * q);
  float4 v[8][2];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (k < splits) {
      v[k][0] = __ldcs(reinterpret_cast<const float4*>(src + k * per_split));
      v[k][1] = __ldcs(reinterpret_cast<const float4*>(src + k * per_split) + 1);
    }
  float4 c0 = dst[0], c1 = dst[1];
  float4 a0 = v[0][0], a1 = v[0][1];
#pragma unroll
  for (int k = 1; k < 8; ++k)
    if (k < splits) {
      a0.x += v[k][0].x; a0.y += v[k][0].y; a0.z += v[k][0].z; a0.w += v[k][0].w;
      a1.x += v[k][1].x; a1.y += v[k][1].y; a1.z += v[k][1].z; a1.w += v[k][1].w;
    }
  c0.x += alpha * a0.x; c0.y += alpha * a0.y; c0.z += alpha * a0.z; c0.w += alpha * a0.w;
  c1.x += alpha * a1.x; c1.y += alpha * a1.y; c1.z += alpha * a1.z; c1.w += alpha * a1.w;
  dst[0] = c0;
  dst[1] = c1;
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

// 2-D tensor map: `inner` contiguous elements per row, `outer` rows, row pitch ld elements.
int encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner, uint64_t outer,
              uint64_t ld, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  PFN_tmapEncodeTiled fn = get_encode_fn();
  if (fn == nullptr) return -3;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (ld * esize) % 16 != 0) return -1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * (uint64_t)esize};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -3;
}
int encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                   uint32_t box_inner, uint32_t box_outer) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, outer, ld, box_inner, box_outer,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}
// Epilogue box map: 32 rows x 64 bytes (32 bf16 or 16 fp32 columns), 64-byte swizzle.
int encode_epi_box(CUtensorMap* map, bool bf16_elems, const void* base, uint64_t cols, uint64_t rows, uint64_t ld) {
  return bf16_elems ? encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, cols, rows, ld, 32, 32,
                                CU_TENSOR_MAP_SWIZZLE_64B)
                    : encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, cols, rows, ld, 16, 32,
                                CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int BN, bool A_MN, bool B_MN, int CG, int EK>
int launch_tc(cudaStream_t st, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tout,
              const CUtensorMap& tin, const CUtensorMap& tout2, TileSched sched, const EpiParams& ep, int num_sms) {
  using Cfg = TileCfg<BN, CG, EK == EK_RESID>;
  auto kern = gemm_tc_kernel<BN, A_MN, B_MN, CG, EK>;
  // co-resident CTA groups of this kernel on the current device (its shared-memory limit set)
  const int max_groups = per_device_once((const void*)kern, [&]() -> int {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) != cudaSuccess)
      return -3;
    int groups = num_sms / CG;
    if (CG == 2) {
      cudaLaunchConfig_t cfg{};
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * groups);
      cfg.blockDim = dim3(NUM_THREADS);
      cfg.dynamicSmemBytes = Cfg::SMEM;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return -3;
      if (n < groups) groups = n;
    }
    return groups;
  });
  if (max_groups <= 0) return -3;
  const int tiles = sched.m_tiles * sched.n_tiles * sched.splits;
  const int groups = tiles < max_groups ? tiles : max_groups;
  if (CG == 1) {
    kern<<<groups, NUM_THREADS, Cfg::SMEM, st>>>(ta, tb, tout, tin, tout2, sched, ep);
  } else {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * groups);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tout, tin, tout2, sched, ep) != cudaSuccess) return -3;
  }
  note_kernel_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

// launch_tc for the epilogue class of ep.kind
template <int BN, bool A_MN, bool B_MN, int CG>
int launch_tc_ek(cudaStream_t st, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tout,
                 const CUtensorMap& tin, const CUtensorMap& tout2, TileSched sched, const EpiParams& ep, int num_sms) {
  switch (epi_class(ep.kind)) {
    case EK_RESID: return launch_tc<BN, A_MN, B_MN, CG, EK_RESID>(st, ta, tb, tout, tin, tout2, sched, ep, num_sms);
    case EK_GELU_FWD:
      return launch_tc<BN, A_MN, B_MN, CG, EK_GELU_FWD>(st, ta, tb, tout, tin, tout2, sched, ep, num_sms);
    case EK_GELU_BWD:
      return launch_tc<BN, A_MN, B_MN, CG, EK_GELU_BWD>(st, ta, tb, tout, tin, tout2, sched, ep, num_sms);
    case EK_CE: return launch_tc<BN, A_MN, B_MN, CG, EK_CE>(st, ta, tb, tout, tin, tout2, sched, ep, num_sms);
    case EK_PLAIN: return launch_tc<BN, A_MN, B_MN, CG, EK_PLAIN>(st, ta, tb, tout, tin, tout2, sched, ep, num_sms);
    default: return launch_tc<BN, A_MN, B_MN, CG, EK_F32>(st, ta, tb, tout, tin, tout2, sched, ep, num_sms);
  }
}

}  // namespace

int gemm_tc_tile_n(int N) { return N > 128 ? 256 : 128; }
int gemm_tc_ce_tiles(int N) { return cdiv(N, gemm_tc_tile_n(N)) * 2; }

namespace {
// Picks the output tile width (128, 192 or 256 columns), the CTA group (one CTA per
// 128-row tile, or a CTA pair per 256-row tile) and the number of K splits from a small
// cost model in MMA clock cycles: the busiest SM's tiles x the tile's main loop (narrower
// tiles re-read more operand bytes per FLOP, hence the efficiency factor; a pair stages half
// the operand bytes per SM and keeps a deeper pipeline), plus for split-K the extra fp32
// traffic of the partials and their reduction.  Pairs are left out where measurement found
// them slower: with split-K, and for the epilogues that read inputs or evaluate GELU on short
// K (the epilogue, not the main loop, bounds those).  GPT2_B200_GEMM_PAIRS=0 / 1 in the
// environment forces single CTAs / pairs (where the shape allows them).
struct TileChoice {
  int bn, splits, cg;
};
TileChoice choose_tiles(int M, int N, int K, bool can_split, size_t ws_elems, int num_sms, bool fixed_bn,
                        bool a_mn, bool b_mn, bool heavy_epilogue) {
  const int nk = cdiv(K, BK);
  const int bns[3] = {256, 192, 128};
  const double eff[3] = {1.0, 0.96, 0.88};
  const char* env = getenv("GPT2_B200_GEMM_PAIRS");
  const int pairs = (env && env[0] == '0') ? 0 : ((env && env[0] == '1') ? 1 : -1);
  TileChoice best{gemm_tc_tile_n(N), 1, 1};
  double best_cost = 1e300;
  for (int cg = 1; cg <= 2; ++cg) {
    if (cg == 2 && (pairs == 0 || M <= BM)) continue;
    if (cg == 2 && pairs != 1 && heavy_epilogue && K < 1536) continue;
    if (cg == 1 && pairs == 1 && M > BM) continue;
    for (int i = 0; i < 3; ++i) {
      const int bn = bns[i];
      if (fixed_bn && bn != gemm_tc_tile_n(N)) continue;
      if (bn > 128 && N <= 128) continue;
      if (cg == 2 && b_mn && bn == 192) continue;   // MN-major B is staged in 64-column boxes
      const int tiles = cdiv(M, BM * cg) * cdiv(N, bn);
      // Weight gradients (both operands MN-major, K = tokens): narrower tiles issue more L2
      // requests per MMA clock and run slower than the single-CTA model says, and large ones
      // may split K on CTA pairs, whose halved operand traffic outweighs the partial sums.
      // Measured over 16384 tokens: 768 x 3072 and 3072 x 768 take 66-68 us as 256-column
      // pairs split in two, 74 us as 256-column single CTAs split in two, 91-96 us as 128-column
      // tiles (single or pairs); 2304 x 768 takes 59 us as pairs split in two against 63 us.
      const bool dw_pairs = a_mn && b_mn && (long long)M * N >= (1LL << 20);
      if (cg == 2 && pairs != 1 && tiles < num_sms / 2 && !dw_pairs) continue;   // pairs only with a full wave of tiles
      for (int sp = 1; sp <= (can_split ? 8 : 1); ++sp) {
        if (sp > 1 && (nk / sp < 8 || N % 4 != 0 || (size_t)sp * cdiv(M, BM * cg) * BM * cg * N > ws_elems)) break;
        if (sp > 1 && cg == 2 && pairs != 1 && !dw_pairs) break;
        if (cg == 2 && pairs != 1 && dw_pairs && tiles * sp * 10 < (num_sms / 2) * 7) continue;   // most of a wave
        if (cg == 2 && pairs != 1 && dw_pairs && sp > 2) break;   // splits measured: 1 and 2
        const int kb = cdiv(nk, sp);
        // MMA clocks per SM of a (128 cg) x bn x 64kb tile + overhead
        const double eff_i = dw_pairs ? (bn == 256 ? 1.0 : (bn == 192 ? 0.88 : 0.62)) : eff[i];
        const double per_tile = ((double)bn * kb * 2.0 / eff_i + 1500.0) / (cg == 2 ? 1.2 : 1.0);
        const double waves = (double)cdiv(tiles * sp, num_sms / cg);
        double cost = waves * per_tile;
        if (sp > 1) cost += (double)(sp + 2) * M * N * 4.0 / 6.0e12 * 1.9e9 + 3000.0;   // partial traffic + reduce launch
        if (cost < best_cost * 0.999) {
          best_cost = cost;
          best = TileChoice{bn, sp, cg};
        }
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
  const bool can_split = (ep.kind == EPI_ACCUM_F32 && ws != nullptr && (reinterpret_cast<uintptr_t>(ep.C) % 16) == 0 &&
                         (reinterpret_cast<uintptr_t>(ws) % 16) == 0);
  // the softmax partials of EPI_CE_FWD are laid out per 256/128-column tile
  const bool heavy = (ep.kind == EPI_RESID_F32 || ep.kind == EPI_GELU_FWD || ep.kind == EPI_GELU_BWD ||
                     ep.kind == EPI_CE_FWD);
  const TileChoice tc = choose_tiles(M, N, K, can_split, ws_elems, num_sms, ep.kind == EPI_CE_FWD, a_mn, b_mn,
                                     heavy);
  const int BN = tc.bn;
  const int CG = tc.cg;
  CUtensorMap ta, tb;
  int rc;
  if (!a_mn) rc = encode_bf16_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda, BK, BM);
  else rc = encode_bf16_2d(&ta, A, (uint64_t)M, (uint64_t)K, (uint64_t)lda, 64, BK);
  if (rc) return rc;
  if (!b_mn) rc = encode_bf16_2d(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)ldb, BK, (uint32_t)(BN / CG));
  else rc = encode_bf16_2d(&tb, B, (uint64_t)N, (uint64_t)K, (uint64_t)ldb, 64, BK);
  if (rc) return rc;

  TileSched sched;
  sched.m_tiles = cdiv(M, BM * CG);
  sched.n_tiles = cdiv(N, BN);
  sched.nk = cdiv(K, BK);
  sched.splits = 1;
  sched.kb_per_split = sched.nk;
  sched.n_fast = sched.n_tiles <= 8 ? 1 : 0;
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
  // epilogue tensor maps: output, input (residual / accumulator / GELU pre-activation),
  // second output (GELU pre-activation); unused ones repeat the output map
  CUtensorMap tout, tin, tout2;
  const int Mpad = cdiv(M, BM * CG) * BM * CG;
  if (split) {
    run.ld_aux = Mpad;   // rows per split in the workspace
    rc = encode_epi_box(&tout, false, ws, (uint64_t)N, (uint64_t)sched.splits * Mpad, (uint64_t)N);
  } else {
    const bool ob = (ep.kind == EPI_STORE_ACT || ep.kind == EPI_GELU_FWD || ep.kind == EPI_GELU_BWD ||
                     ep.kind == EPI_CE_FWD);
    rc = encode_epi_box(&tout, ob, ep.C, (uint64_t)N, (uint64_t)M, (uint64_t)ep.ldc);
  }
  if (rc) return rc;
  tin = tout;
  tout2 = tout;
  if (!split && ep.kind == EPI_RESID_F32)
    rc = encode_epi_box(&tin, false, ep.aux, (uint64_t)N, (uint64_t)M, (uint64_t)ep.ld_aux);
  else if (!split && ep.kind == EPI_GELU_BWD)
    rc = encode_epi_box(&tin, true, ep.aux, (uint64_t)N, (uint64_t)M, (uint64_t)ep.ld_aux);
  if (rc) return rc;
  if (ep.kind == EPI_GELU_FWD)
    rc = encode_epi_box(&tout2, true, ep.aux_out, (uint64_t)N, (uint64_t)M, (uint64_t)ep.ld_aux_out);
  if (rc) return rc;
#define LAUNCH_BN(BNV, CGV)                                                                                   \
  do {                                                                                                        \
    if (!a_mn && !b_mn) rc = launch_tc_ek<BNV, false, false, CGV>(st, ta, tb, tout, tin, tout2, sched, run, num_sms);   \
    else if (!a_mn && b_mn) rc = launch_tc_ek<BNV, false, true, CGV>(st, ta, tb, tout, tin, tout2, sched, run, num_sms); \
    else rc = launch_tc_ek<BNV, true, true, CGV>(st, ta, tb, tout, tin, tout2, sched, run, num_sms);                    \
  } while (0)
  if (CG == 1) {
    if (BN == 256) LAUNCH_BN(256, 1);
    else if (BN == 192) LAUNCH_BN(192, 1);
    else LAUNCH_BN(128, 1);
  } else {
    if (BN == 256) LAUNCH_BN(256, 2);
    else if (BN == 192) {
      if (b_mn) return -1;   // excluded by the tile choice
      rc = launch_tc_ek<192, false, false, 2>(st, ta, tb, tout, tin, tout2, sched, run, num_sms);
    } else LAUNCH_BN(128, 2);
  }
#undef LAUNCH_BN
  if (rc) return rc;
  if (split && N % 8 == 0 && ep.ldc % 8 == 0) {
    const long long total = (long long)M * (N / 8);
    splitk_reduce8_kernel<<<(unsigned)cdivll(total, 256), 256, 0, st>>>(reinterpret_cast<float*>(ep.C), ep.ldc, ws,
                                                                       M, Mpad, N, sched.splits, ep.alpha);
    note_kernel_launches(1);
    if (cudaGetLastError() != cudaSuccess) return -3;
  } else if (split) {
    const long long total = (long long)M * (N / 4);
    const int threads = 256;
    long long nb = cdivll(total, threads);
    if (nb > (long long)num_sms * 8) nb = (long long)num_sms * 8;
    const int blocks = (int)nb;
    splitk_reduce_kernel<<<blocks, threads, 0, st>>>(reinterpret_cast<float*>(ep.C), ep.ldc, ws, M, Mpad, N,
                                                     sched.splits, ep.alpha);
    note_kernel_launches(1);
    if (cudaGetLastError() != cudaSuccess) return -3;
  }
  return 0;
}
