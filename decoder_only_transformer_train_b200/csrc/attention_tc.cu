// Causal flash-attention forward on the sm_100a tensor cores (head size 64, bf16).
//
// "Karpathy's Zero to Hero, Lecture 9" notes, "2:00:19 – 2:06:39 FlashAttention": the
// scores, mask, softmax and weighted sum fused in one kernel that never writes the T x T
// matrix, using the online softmax (running max and sum).
//
// Persistent: one CTA per SM walks (batch, head, 128-query tile) items, heaviest (latest)
// query tiles first; Q is double-buffered so the pipeline runs on across items.
//   warp 0      : TMA producer - Q of each item, then its K_j / V_j tiles of 128 keys,
//                 all straight out of the qkv activation [B*T, 3C]
//   warp 1      : TMEM allocator + MMA issuer:  S_j = Q K_j^T    (128 x 128, TMEM)
//                                                O  += P_j V_j    (128 x 64, TMEM)
//   warps 2..9  : two softmax groups of four warps; the CTA's key tiles alternate between
//                 them (global tile counter parity).  Thread r of a group owns query row r
//                 (= TMEM lane r): it reads S_j, applies the causal mask, and writes
//                 P_j = 2^(s*log2e/sqrt(hd) - m_ref) as bf16 pairs into the group's P columns
//                 of TMEM, from where the P V product reads it as its A operand.  Each group
//                 accumulates its own O in TMEM; m_ref only moves when a row's max grows by
//                 more than 2^8, and then the thread rescales its O row in TMEM before the
//                 next MMA.  At the end of an item the two groups' (m_ref, l, O) are merged.
#include <math.h>
#include <stdlib.h>
#include <type_traits>
#include "sm100.cuh"
#include "kernels.h"

namespace {

constexpr int QT = 128;          // queries per item
constexpr int KT = 128;          // keys per tile
constexpr int HD = 64;
constexpr int KV_STAGES = 5;
constexpr int NUM_THREADS = 320;
constexpr int TILE_BYTES = KT * HD * 2;        // 16 KB: one Q, K or V tile
constexpr int SMEM_BYTES = 2 * TILE_BYTES + 2 * KV_STAGES * TILE_BYTES + QT * 8 + 512 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0;                  // S of group g: columns [128 g, 128 g + 128)
constexpr uint32_t O_COL = 256;                // O of group g: columns [256 + 64 g, 256 + 64 g + 64)
constexpr uint32_t P_COL = 384;                // P of group g (bf16 pairs): columns [384 + 64 g, 384 + 64 g + 64)
constexpr float RESCALE_THRESHOLD = 8.0f;      // log2 units


// Row max over the first 32 columns of an S tile in TMEM; on the diagonal tile the keys after
// query row r are left out (key 0 never is).
template <bool DIAG>
__device__ __forceinline__ float s_chunk32_max(uint32_t taddr, int r) {
  uint32_t v[32];
  tmem_ld32(taddr, v);
  tmem_wait_ld_regs(v);
  float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float a = __uint_as_float(v[e]), b = __uint_as_float(v[e + 1]);
    if (DIAG) {
      if (e > r) a = -INFINITY;
      if (e + 1 > r) b = -INFINITY;
    }
    m4[(e >> 1) & 3] = max3f(m4[(e >> 1) & 3], a, b);
  }
  return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
}

// P = 2^(s * scale_log2 - m_ref) for a 128-column S row, written as bf16 pairs into the 64
// P columns at TMEM address pcol (this thread's lane); returns the row sum of P (four
// independent partial sums).  With MAX, the same pass also returns the row's raw max in *mx
// (masked keys left out), so that a tile whose max stays within the rescale threshold of m_ref
// is read from TMEM once.  The row goes in 16-column chunks, the next chunk's TMEM load in
// flight while the current one is computed (the loop over chunk pairs is kept rolled, which
// keeps the pipeline within the registers).
template <bool DIAG, bool MAX = false>
__device__ __forceinline__ float p_row_store(uint32_t taddr, int r, float scale_log2, float m_ref, uint32_t pcol,
                                             float* mx = nullptr) {
  float2 sum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  const float2 sc = make_float2(scale_log2, scale_log2);
  const float2 nm = make_float2(-m_ref, -m_ref);
  // on the diagonal tile rows below 64 (warps of lane quarters 0 and 1; warp-uniform) have no
  // unmasked key in the second half: P is zero there
  const int nch = (DIAG && r < 64) ? 4 : 8;   // 16-column chunks holding unmasked keys
  uint32_t w[16];
  auto chunk = [&](int c0, const uint32_t (&v)[16]) {
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const float sa = __uint_as_float(v[e]), sb = __uint_as_float(v[e + 1]);
      const float2 x = ffma2(make_float2(sa, sb), sc, nm);
      float pa = ex2(x.x), pb = ex2(x.y);
      if (DIAG) {
        const int col = c0 + e;
        if (col > r) pa = 0.f;
        if (col + 1 > r) pb = 0.f;
      }
      if (MAX) {
        const int col = c0 + e;
        const float ma = (DIAG && col > r) ? -INFINITY : sa;
        const float mb = (DIAG && col + 1 > r) ? -INFINITY : sb;
        m4[(e >> 1) & 3] = max3f(m4[(e >> 1) & 3], ma, mb);
      }
      sum[(e >> 1) & 3] = fadd2(sum[(e >> 1) & 3], make_float2(pa, pb));
      w[((c0 & 31) >> 1) + (e >> 1)] = pack_bf16x2(pa, pb);
    }
  };
  uint32_t va[16], vb[16];
  tmem_ld16(taddr, va);
  tmem_wait_ld_regs16(va);
#pragma unroll 1
  for (int c = 0; c < 8; c += 2) {
    if (c < nch) {
      tmem_ld16(taddr + 16 * (c + 1), vb);
      chunk(16 * c, va);
      tmem_wait_ld_regs16(vb);
      if (c + 2 < nch) tmem_ld16(taddr + 16 * (c + 2), va);
      chunk(16 * (c + 1), vb);
      if (c + 2 < nch) tmem_wait_ld_regs16(va);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) w[e] = 0u;
    }
    tmem_st16(pcol + 8 * c, w);
  }
  tmem_wait_st();
  if (MAX) *mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  const float2 s01 = fadd2(sum[0], sum[1]), s23 = fadd2(sum[2], sum[3]);
  return (s01.x + s01.y) + (s23.x + s23.y);
}

// Item order shared by all roles: item t -> (query tile, batch*head), heaviest first.  A
// CTA's k-th item is turn(k): a snake over the grid (turn k takes items k*G .. k*G + G - 1,
// odd turns in reverse), which evens out the item sizes across CTAs (at the 124M shape the
// busiest CTA gets 48 key tiles against 51 when dealt round-robin, for 46.7 on average).
struct FwdItems {
  int n_qt, BH, total;
  __device__ __forceinline__ void get(int t, int& qt, int& bh) const {
    qt = n_qt - 1 - t / BH;
    bh = t % BH;
  }
  __device__ __forceinline__ int turn(int k) const {
    return k * (int)gridDim.x + ((k & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
  }
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse,
                   int B, int T, int H, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                    // [2]
  uint8_t* sK = sQ + 2 * TILE_BYTES;                     // [KV_STAGES]
  uint8_t* sV = sK + KV_STAGES * TILE_BYTES;             // [KV_STAGES]
  float* sML = reinterpret_cast<float*>(sV + KV_STAGES * TILE_BYTES);   // [QT][2]: handed-over (m_ref, l)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sML + 2 * QT);
  uint64_t* q_full = bars;                       // 2
  uint64_t* q_empty = q_full + 2;                // 2
  uint64_t* kv_full = q_empty + 2;               // KV_STAGES
  uint64_t* kv_empty = kv_full + KV_STAGES;      // KV_STAGES
  // S(G) is committed after the group's previous P.V product was issued, so its completion
  // also means that product is done (P columns free, O stable); and the MMA issuer writes a
  // group's next S only after that group's P is in, so its S has been read.  Neither needs a
  // barrier of its own.
  uint64_t* s_full = kv_empty + KV_STAGES;       // 2 (per group)
  uint64_t* p_full = s_full + 2;                 // 2
  uint64_t* o_done = p_full + 2;                 // 2
  uint64_t* merge_full = o_done + 2;             // 1
  uint64_t* merge_empty = merge_full + 1;        // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(merge_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = H * HD;
  FwdItems items{cdiv(T, QT), B * H, cdiv(T, QT) * B * H};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(merge_full, 128);
    mbar_init(merge_empty, 128);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int G = 0;                                   // global key-tile counter
      bool ok = true;
      InflightTx tx{bars, 0u, 0u};
      for (int k = 0, t = items.turn(0); t < items.total && ok; ++k, t = items.turn(k)) {
        int qt, bh;
        items.get(t, qt, bh);
        const int b = bh / H, h = bh % H, row0 = b * T;
        const int qb = k & 1;
        if (!mbar_wait(&q_empty[qb], ((k >> 1) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&q_full[qb], TILE_BYTES);
        tma_load_2d(sQ + qb * TILE_BYTES, &tm_qkv, h * HD, row0 + qt * QT, &q_full[qb]);
        tx.note(&q_full[qb], (k >> 1) & 1);
        for (int j = 0; j <= qt; ++j, ++G) {
          const int s = G % KV_STAGES;
          if (!mbar_wait(&kv_empty[s], ((G / KV_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[s], 2 * TILE_BYTES);
          tma_load_2d(sK + s * TILE_BYTES, &tm_qkv, C + h * HD, row0 + j * KT, &kv_full[s]);
          tma_load_2d(sV + s * TILE_BYTES, &tm_qkv, 2 * C + h * HD, row0 + j * KT, &kv_full[s]);
          tx.note(&kv_full[s], (G / KV_STAGES) & 1);
        }
      }
      if (*abort_flag) tx.drain();   // copies still in flight land before the CTA leaves
    }
  } else if (warp == 1) {
    {
      // ---------------------------------------------------------------- MMA issuer
      // the whole warp runs the loop (its descriptors and counters stay warp-uniform); one
      // elected lane issues the MMAs and commits
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_s = make_idesc_bf16(QT, KT, false, false);   // Q, K both K-major
      constexpr uint32_t idesc_o = make_idesc_bf16(QT, HD, false, true);    // P from TMEM, V MN-major
      // tile iterator over the CTA's flattened (item, j) sequence
      struct It {
        int t, k, qt, j, G;
      };
      auto valid = [&](const It& it) { return it.t < items.total; };
      auto next = [&](It it) {
        ++it.G;
        if (++it.j > it.qt) {
          it.j = 0;
          ++it.k;
          it.t = items.turn(it.k);
          if (it.t < items.total) {
            int bh;
            items.get(it.t, it.qt, bh);
          }
        }
        return it;
      };
      It cur{(int)blockIdx.x, 0, 0, 0, 0};
      if (valid(cur)) {
        int bh;
        items.get(cur.t, cur.qt, bh);
      }
      int co0 = 0, co1 = 0;    // O issues per group
      bool ok = true;
      // operand descriptors of the first Q, K and V buffers; each MMA's is derived by an add
      const uint64_t dQ0 = make_sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = make_sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = make_sdesc_sw128(smem_u32(sV), 8192, 1024);
      auto issue_s = [&](const It& it) -> bool {
        const int g = it.G & 1, s = it.G % KV_STAGES, qb = it.k & 1;
        if (it.j == 0 && !mbar_wait_warp(&q_full[qb], (it.k >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait_warp(&kv_full[s], (it.G / KV_STAGES) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t aQ = sdesc_add(dQ0, qb * TILE_BYTES), bK = sdesc_add(dK0, s * TILE_BYTES);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc_mma_bf16(tmem + S_COL + g * KT, sdesc_add(aQ, kk * 32), sdesc_add(bK, kk * 32), idesc_s,
                        kk > 0 ? 1u : 0u);
          tc_commit(&s_full[g]);
        }
        __syncwarp();
        return true;
      };
      // S of each group's first tile; then per tile: P.V of it and S of the group's next tile
      It nx = next(cur);
      if (valid(cur)) ok = issue_s(cur);
      if (ok && valid(nx)) ok = issue_s(nx);
      while (ok && valid(cur)) {
        const int g = cur.G & 1, s = cur.G % KV_STAGES;
        const int co = g ? co1 : co0;
        if (!mbar_wait_warp(&p_full[g], co & 1, abort_flag)) break;
        if (g) ++co1; else ++co0;
        tc_fence_after();
        const bool first_of_group = (cur.j < 2);          // the group's first tile of this item
        const uint64_t bV = sdesc_add(dV0, s * TILE_BYTES);
        // A: 16 keys of P = 8 TMEM columns per step; B: 16 rows of V, MN-major
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk)
            tc_mma_bf16_ts(tmem + O_COL + g * HD, tmem + P_COL + g * 64 + kk * 8, sdesc_add(bV, kk * 2048), idesc_o,
                           (kk > 0 || !first_of_group) ? 1u : 0u);
          tc_commit(&kv_empty[s]);
          if (cur.j + 2 > cur.qt) tc_commit(&o_done[g]);    // the group's last tile of this item
          if (cur.j == cur.qt) tc_commit(&q_empty[cur.k & 1]);
        }
        __syncwarp();
        const It n2 = next(nx);                           // the same group's next tile
        if (valid(n2) && !issue_s(n2)) break;
        cur = nx;
        nx = n2;
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int grp = (warp - 2) >> 2;             // key tiles with global counter parity grp
    const int q = warp & 3;
    const int r = q * 32 + lane;                 // query row within the item
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t s_col = S_COL + grp * KT;
    const uint32_t pcol = tmem + lane_off + P_COL + grp * 64;   // this row's P columns
    int c = 0, d = 0, hcount = 0;                // this group's tiles, items, handovers
    bool pending = false;                        // an O handover the finisher has not released yet
    bool ok = true;
    int G = 0;
    for (int k = 0, t = items.turn(0); t < items.total && ok; ++k, t = items.turn(k)) {
      int qt, bh;
      items.get(t, qt, bh);
      const int n_kv = qt + 1;
      const int G0 = G;
      G += n_kv;
      float m_ref = -INFINITY, l = 0.f;
      bool has = false;
      for (int j = ((G0 & 1) == grp) ? 0 : 1; j < n_kv; j += 2) {
        if (!mbar_wait_warp(&s_full[grp], c & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool diag = (j == qt);
        const uint32_t srow = tmem + lane_off + s_col;
        float sum;
        if (!has) {
          // the group's first tile of the item: a first m_ref from the row's max over the tile's
          // first 32 keys (on the diagonal tile key 0 is always valid); the pass below tracks
          // the true max and writes P again if it grew past the threshold
          m_ref = (diag ? s_chunk32_max<true>(srow, r) : s_chunk32_max<false>(srow, r)) * scale_log2;
        }
        // one pass: P against the current m_ref, and the tile's row max alongside
        float mx;
        sum = diag ? p_row_store<true, true>(srow, r, scale_log2, m_ref, pcol, &mx)
                   : p_row_store<false, true>(srow, r, scale_log2, m_ref, pcol, &mx);
        const float m_new = mx * scale_log2;
        const bool grow = m_new > m_ref + RESCALE_THRESHOLD;
        // tcgen05.ld / st are warp-collective, so the whole warp takes this branch when any of
        // its rows' max grew past the threshold: those rows rescale O (from the item's second
        // tile of the group on; before it O holds nothing of this item) and l and write P again
        // against the new max; the others scale by exactly 1 and write the same P again.
        if (__any_sync(0xffffffffu, grow)) {
          const float f = grow ? ex2(m_ref - m_new) : 1.0f;
          if (has) {
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < HD; c0 += 16) {
              uint32_t v[16];
              tmem_ld16(tmem + lane_off + O_COL + grp * HD + c0, v);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
              tmem_st16(tmem + lane_off + O_COL + grp * HD + c0, v);
            }
            tmem_wait_st();
          }
          l *= f;
          if (grow) m_ref = m_new;
          sum = diag ? p_row_store<true>(srow, r, scale_log2, m_ref, pcol)
                     : p_row_store<false>(srow, r, scale_log2, m_ref, pcol);
        }
        l += sum;
        tc_fence_before();
        // an O row handed over at the previous item must be read before this group's next MMA
        if (pending) {
          if (!mbar_wait_warp(merge_empty, (hcount & 1) ^ 1, abort_flag)) { ok = false; break; }
          pending = false;
        }
        mbar_arrive(&p_full[grp]);   // P is in TMEM (tcgen05.wait::st, then the fence above)
        has = true;
        ++c;
      }
      if (!ok) break;
      if (has) {
        if (!mbar_wait_warp(&o_done[grp], d & 1, abort_flag)) { ok = false; break; }
        ++d;
      }
      const int finisher = (G0 + n_kv - 1) & 1;
      const bool both = n_kv >= 2;
      if (grp != finisher) {
        if (both) {
          // hand (m_ref, l) over; O stays in this group's TMEM columns for the finisher
          if (pending && !mbar_wait_warp(merge_empty, (hcount & 1) ^ 1, abort_flag)) { ok = false; break; }
          sML[r * 2] = m_ref;
          sML[r * 2 + 1] = l;
          mbar_arrive(merge_full);
          pending = true;
          ++hcount;
        }
      } else {
        const int qi = qt * QT + r;
        float m1 = -INFINITY, l1 = 0.f;
        if (both) {
          if (!mbar_wait_warp(merge_full, hcount & 1, abort_flag)) { ok = false; break; }
          m1 = sML[r * 2];
          l1 = sML[r * 2 + 1];
        }
        tc_fence_after();
        const float M = fmaxf(m_ref, m1);
        const float a0 = ex2(m_ref - M), a1 = both ? ex2(m1 - M) : 0.f;
        const float inv = 1.0f / (l * a0 + l1 * a1);
        const int b = bh / H, h = bh % H;
        bf16* orow = out + (long long)(b * T + qi) * C + h * HD;
#pragma unroll 1
        for (int c0 = 0; c0 < HD; c0 += 16) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tmem + lane_off + O_COL + grp * HD + c0, v0);
          if (both) tmem_ld16(tmem + lane_off + O_COL + (grp ^ 1) * HD + c0, v1);
          tmem_wait_ld();
          if (qi < T) {
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
              float o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int idx = g8 * 8 + e;
                o[e] = (__uint_as_float(v0[idx]) * a0 + (both ? __uint_as_float(v1[idx]) * a1 : 0.f)) * inv;
              }
              uint4 w;
              w.x = pack_bf16x2(o[0], o[1]);
              w.y = pack_bf16x2(o[2], o[3]);
              w.z = pack_bf16x2(o[4], o[5]);
              w.w = pack_bf16x2(o[6], o[7]);
              reinterpret_cast<uint4*>(orow + c0)[g8] = w;
            }
          }
        }
        if (qi < T) lse[(long long)bh * T + qi] = (M + log2f(l * a0 + l1 * a1)) * 0.6931471805599453f;
        if (both) {
          tc_fence_before();
          mbar_arrive(merge_empty);
          ++hcount;
        }
      }
    }
    if (ok && pending) mbar_wait_warp(merge_empty, (hcount & 1) ^ 1, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

typedef CUresult (*PFN_encode)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encode encode_fn() {
  static PFN_encode fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encode>(p);
  }
  return fn;
}

}  // namespace

// Tensor-core forward for head size 64 in bf16; returns -4 when the shape is not covered.
int launch_attn_fwd_tc(cudaStream_t st, const void* qkv, void* out, float* lse, int B, int T, int H, int hd) {
  if (hd != HD) return -4;
  const int C = H * HD;
  PFN_encode fn = encode_fn();
  if (fn == nullptr) return -3;
  // TMA reads qkv; the epilogue writes out with 16-byte stores
  if (((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15) != 0) return -1;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)(3 * C), (cuuint64_t)B * T};
  cuuint64_t strides[1] = {(cuuint64_t)(3 * C) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(qkv), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return -3;
  const int nsm = current_device_sms();
  const int total = cdiv(T, QT) * B * H;
  const int grid = total < nsm ? total : nsm;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  if (set_dynamic_smem_once((const void*)attn_fwd_tc_kernel, SMEM_BYTES)) return -3;
  attn_fwd_tc_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tm, reinterpret_cast<bf16*>(out), lse, B, T, H,
                                                            scale_log2);
  note_kernel_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

// ============================================================================ backward
// Gradients of the causal attention with the probabilities recomputed from the saved
// log-sum-exp (scaled scores z = q.k / sqrt(hd), P = softmax(z), D = rowsum(dO * O)):
//   dV = P^T dO,   dZ = P * (dO V^T - D),   dQ = dZ K / sqrt(hd),   dK = dZ^T Q / sqrt(hd).
// Two kernels keep every sum in a fixed order (no atomics): the dK/dV kernel accumulates
// each 128-key tile over the query tiles at or after it, the dQ kernel each 128-query tile
// over the key tiles at or before it.  P and dZ never leave the SM: the elementwise warps
// write them as bf16 into tensor memory, from where the MMAs read them as their A operand.
namespace {

constexpr int BWD_THREADS = 576;   // producer, MMA, 16 elementwise warps (4 per TMEM lane quarter)
constexpr int BWD_STAGES = 4;
// smem: two buffers of the 2 resident tiles (K_j,V_j or Q_i,dO_i: this item's and the next
// one's), BWD_STAGES x 2 streamed tiles, per-warp column scalars and barriers
constexpr int BWD_VEC_BYTES = 16 * 64 * 4;
constexpr int BWD_SMEM = 4 * TILE_BYTES + BWD_STAGES * 2 * TILE_BYTES + BWD_VEC_BYTES + 512 + 1024;
static_assert(BWD_SMEM <= 232448, "attention backward shared memory");
// TMEM columns: S [0,128) and dP [128,256) in fp32; P [256,320) and dZ [320,384) as bf16 pairs;
// accumulators from 384: the dK/dV kernel's dV [384,448) and dK [448,512), the dQ kernel's dQ
// in two buffers [384,448) and [448,512)
constexpr uint32_t BS_C = 0, BDP_C = 128, BP_C = 256, BDS_C = 320, BACC_C = 384;

// Work items of the backward: (128-row tile, batch*head), heaviest first.
//   MODE 0 (dK/dV): item = key tile j, streams the query tiles i >= j  (n_t - j of them)
//   MODE 1 (dQ):    item = query tile i, streams the key tiles j <= i  (i + 1 of them)
struct BwdItem {
  int tile, bh, it0, it1;
};
template <int MODE>
__device__ __forceinline__ BwdItem bwd_item(int idx, int BH, int n_t) {
  BwdItem w;
  w.tile = (MODE == 0) ? idx / BH : n_t - 1 - idx / BH;
  w.bh = idx % BH;
  w.it0 = (MODE == 0) ? w.tile : 0;
  w.it1 = (MODE == 0) ? n_t : w.tile + 1;
  return w;
}
// Item of a CTA's k-th turn: a snake over the grid (turn k takes items k*G .. k*G + G - 1,
// odd turns in reverse), which evens out the heaviest-first item sizes across CTAs.
__device__ __forceinline__ int bwd_turn_item(int k) {
  return k * (int)gridDim.x + ((k & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
}

// MODE 0: dK/dV kernel, a key per TMEM lane: S^T = K_j Q_i^T and dP^T = V_j dO_i^T, then
//         dV += P^T dO_i and dK += dZ^T Q_i with P^T and dZ^T read from TMEM.
// MODE 1: dQ kernel, a query per TMEM lane: S = Q_i K_j^T and dP = dO_i V_j^T, then
//         dQ += dZ K_j with dZ read from TMEM.
// Persistent: each CTA walks its items in turn.  Resident tiles are double-buffered across
// items (and the dQ accumulator too), so the next item's loads and first S / dP products
// overlap the current item's last tile and epilogue.
// With bias_part non-null the epilogue also writes column sums of the gradients it produces
// (the bias gradient of c_attn, before the bf16 rounding of dqkv): row (tile * B + b) * 4 + q,
// columns [0, 3C), sums over the 32 rows of TMEM lane quarter q of the 128-row tile; every
// (row, column) is written by exactly one item of one of the two kernels.
template <int MODE>
__global__ void __launch_bounds__(BWD_THREADS, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                   const float* __restrict__ lse, const float* __restrict__ Dbuf, bf16* __restrict__ dqkv,
                   float* __restrict__ bias_part, int B, int T, int H, float scale, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRes = smem;                                  // [2][K_j,V_j (MODE 0) / Q_i,dO_i (MODE 1)]
  uint8_t* sA = sRes + 4 * TILE_BYTES;                   // streamed: Q_i (MODE 0) / K_j (MODE 1)
  uint8_t* sB = sA + BWD_STAGES * TILE_BYTES;            // streamed: dO_i (MODE 0) / V_j (MODE 1)
  float* sVec = reinterpret_cast<float*>(sB + BWD_STAGES * TILE_BYTES);   // [16 warps][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sVec) + BWD_VEC_BYTES);
  uint64_t* r_full = bars;                               // [2] resident tiles loaded
  uint64_t* r_empty = r_full + 2;                        // [2] resident tiles no longer read
  uint64_t* t_full = r_empty + 2;                        // [BWD_STAGES]
  uint64_t* t_empty = t_full + BWD_STAGES;               // [BWD_STAGES]
  uint64_t* sd_full = t_empty + BWD_STAGES;              // S and dP in TMEM
  uint64_t* s_empty = sd_full + 1;                       // S read out
  uint64_t* dp_empty = s_empty + 1;                      // dP read out
  uint64_t* ps_full = dp_empty + 1;                      // P and dZ written to TMEM
  uint64_t* ps_empty = ps_full + 1;                      // P and dZ consumed by the MMAs
  uint64_t* acc_full = ps_empty + 1;                     // [2] an item's accumulation done
  uint64_t* acc_empty = acc_full + 2;                    // [2] an item's accumulators read out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_t = cdiv(T, 128);
  const int BH = B * H;
  const int n_items = n_t * BH;
  const int C = H * HD;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&r_full[i], 1);
      mbar_init(&r_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 512);
    }
    for (int i = 0; i < BWD_STAGES; ++i) {
      mbar_init(&t_full[i], 1);
      mbar_init(&t_empty[i], 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(s_empty, 512);
    mbar_init(dp_empty, 512);
    mbar_init(ps_full, 512);
    mbar_init(ps_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int g = 0;   // streamed tiles issued by this CTA (stage ring position)
      InflightTx tx{bars, 0u, 0u};
      for (int k = 0;; ++k) {
        const int idx = bwd_turn_item(k);
        if (idx >= n_items) break;
        const BwdItem w = bwd_item<MODE>(idx, BH, n_t);
        const int row0 = (w.bh / H) * T, h = w.bh % H;
        const int rb = k & 1;
        if (!mbar_wait(&r_empty[rb], ((k >> 1) & 1) ^ 1, abort_flag)) break;
        uint8_t* r0 = sRes + rb * 2 * TILE_BYTES;
        mbar_arrive_expect_tx(&r_full[rb], 2 * TILE_BYTES);
        if (MODE == 0) {
          tma_load_2d(r0, &tm_qkv, C + h * HD, row0 + w.tile * 128, &r_full[rb]);                  // K_j
          tma_load_2d(r0 + TILE_BYTES, &tm_qkv, 2 * C + h * HD, row0 + w.tile * 128, &r_full[rb]);  // V_j
        } else {
          tma_load_2d(r0, &tm_qkv, h * HD, row0 + w.tile * 128, &r_full[rb]);                      // Q_i
          tma_load_2d(r0 + TILE_BYTES, &tm_do, h * HD, row0 + w.tile * 128, &r_full[rb]);           // dO_i
        }
        tx.note(&r_full[rb], (k >> 1) & 1);
        bool ok = true;
        for (int t = w.it0; t < w.it1; ++t, ++g) {
          const int st = g % BWD_STAGES;
          if (!mbar_wait(&t_empty[st], ((g / BWD_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&t_full[st], 2 * TILE_BYTES);
          if (MODE == 0) {
            tma_load_2d(sA + st * TILE_BYTES, &tm_qkv, h * HD, row0 + t * 128, &t_full[st]);          // Q_i
            tma_load_2d(sB + st * TILE_BYTES, &tm_do, h * HD, row0 + t * 128, &t_full[st]);           // dO_i
          } else {
            tma_load_2d(sA + st * TILE_BYTES, &tm_qkv, C + h * HD, row0 + t * 128, &t_full[st]);      // K_j
            tma_load_2d(sB + st * TILE_BYTES, &tm_qkv, 2 * C + h * HD, row0 + t * 128, &t_full[st]);  // V_j
          }
          tx.note(&t_full[st], (g / BWD_STAGES) & 1);
        }
        if (!ok) break;
      }
      if (*abort_flag) tx.drain();   // copies still in flight land before the CTA leaves
    }
  } else if (warp == 1) {
    {
      // ---------------------------------------------------------------- MMA issuer
      // the whole warp runs the loop (descriptors and counters stay warp-uniform); one elected
      // lane issues the MMAs and commits
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_sq = make_idesc_bf16(128, 128, false, false);   // 128x128, K=64, both K-major
      constexpr uint32_t idesc_acc = make_idesc_bf16(128, HD, false, true);    // 128x64, K=128: A from TMEM,
                                                                               // B MN-major
      // S / dP of the CTA's g-th streamed tile, read against resident buffer rb: the resident
      // tiles are the A operands in MODE 0 (rows: keys) and in MODE 1 (rows: queries)
      // operand descriptors of the first buffers (K-major for S / dP, MN-major for the
      // accumulations); each MMA's is derived by an add
      const uint64_t dA_k = make_sdesc_sw128(smem_u32(sA), 16, 1024), dA_mn = make_sdesc_sw128(smem_u32(sA), 8192, 1024);
      const uint64_t dB_k = make_sdesc_sw128(smem_u32(sB), 16, 1024), dB_mn = make_sdesc_sw128(smem_u32(sB), 8192, 1024);
      const uint64_t dR_k = make_sdesc_sw128(smem_u32(sRes), 16, 1024);
      auto issue_sd = [&](int g, int rb) -> bool {
        const int st = g % BWD_STAGES;
        if (!mbar_wait_warp(&t_full[st], (g / BWD_STAGES) & 1, abort_flag)) return false;
        // S goes as soon as the elementwise warps have read the previous S, dP once they have
        // read the previous dP (its second half comes after their first half's arithmetic)
        if (!mbar_wait_warp(s_empty, (g & 1) ^ 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t a = sdesc_add(dA_k, st * TILE_BYTES), bq = sdesc_add(dB_k, st * TILE_BYTES);
        const uint64_t r0 = sdesc_add(dR_k, rb * 2 * TILE_BYTES), r1 = sdesc_add(r0, TILE_BYTES);
        if (leader) {
#pragma unroll
          for (int k = 0; k < HD / 16; ++k)   // MODE 0: S^T = K_j Q_i^T;  MODE 1: S = Q_i K_j^T
            tc_mma_bf16(tmem + BS_C, sdesc_add(r0, k * 32), sdesc_add(a, k * 32), idesc_sq, k > 0 ? 1u : 0u);
        }
        __syncwarp();
        if (!mbar_wait_warp(dp_empty, (g & 1) ^ 1, abort_flag)) return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < HD / 16; ++k)   // MODE 0: dP^T = V_j dO_i^T;  MODE 1: dP = dO_i V_j^T
            tc_mma_bf16(tmem + BDP_C, sdesc_add(r1, k * 32), sdesc_add(bq, k * 32), idesc_sq, k > 0 ? 1u : 0u);
          tc_commit(sd_full);
        }
        __syncwarp();
        return true;
      };
      bool ok = true;
      int g = 0;
      int idx = bwd_turn_item(0);
      if (idx < n_items) ok = mbar_wait_warp(&r_full[0], 0, abort_flag) && issue_sd(0, 0);
      for (int k = 0; idx < n_items && ok; ++k) {
        const BwdItem w = bwd_item<MODE>(idx, BH, n_t);
        const int n_it = w.it1 - w.it0;
        const int nidx = bwd_turn_item(k + 1);
        const int ab = (MODE == 0) ? 0 : (k & 1);            // dK/dV: one accumulator buffer; dQ: two
        const uint32_t acc0 = tmem + BACC_C + ab * 64, acc1 = acc0 + 64;
        for (int n = 0; n < n_it && ok; ++n, ++g) {
          // S / dP one tile ahead, possibly the next item's first
          if (n + 1 < n_it) {
            ok = issue_sd(g + 1, k & 1);
          } else if (nidx < n_items) {
            ok = mbar_wait_warp(&r_full[(k + 1) & 1], ((k + 1) >> 1) & 1, abort_flag) && issue_sd(g + 1, (k + 1) & 1);
          }
          if (!ok) break;
          // the accumulator buffer must have been read out by the epilogue of the item that
          // last used it (item k - 1 for dK/dV, k - 2 for dQ)
          if (n == 0) {
            const bool got = (MODE == 0) ? mbar_wait_warp(&acc_empty[0], (k & 1) ^ 1, abort_flag)
                                         : mbar_wait_warp(&acc_empty[ab], ((k >> 1) & 1) ^ 1, abort_flag);
            if (!got) { ok = false; break; }
          }
          const int st = g % BWD_STAGES;
          if (!mbar_wait_warp(ps_full, g & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a = sdesc_add(dA_mn, st * TILE_BYTES), bq = sdesc_add(dB_mn, st * TILE_BYTES);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t accum = (n > 0 || kk > 0) ? 1u : 0u;
              // A: 16 queries (MODE 0) or keys (MODE 1) of P / dZ = 8 TMEM columns per step;
              // B: the same 16 rows of a [128 x 64] tile, MN-major (2 KB per step)
              if (MODE == 0) {
                tc_mma_bf16_ts(acc0, tmem + BP_C + kk * 8, sdesc_add(bq, kk * 2048), idesc_acc, accum);   // dV += P^T dO_i
                tc_mma_bf16_ts(acc1, tmem + BDS_C + kk * 8, sdesc_add(a, kk * 2048), idesc_acc, accum);   // dK += dZ^T Q_i
              } else {
                tc_mma_bf16_ts(acc0, tmem + BDS_C + kk * 8, sdesc_add(a, kk * 2048), idesc_acc, accum);   // dQ += dZ K_j
              }
            }
            tc_commit(&t_empty[st]);
            tc_commit(ps_empty);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (leader) {
          tc_commit(&acc_full[ab]);
          tc_commit(&r_empty[k & 1]);
        }
        __syncwarp();
        idx = nidx;
      }
    }
  } else {
    // ------------------------------------------------------------------ elementwise
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;            // columns [32*part, 32*part + 32) of each tile
    const int r = q * 32 + lane;                 // TMEM lane: a key (MODE 0) or a query (MODE 1)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float LOG2E = 1.4426950408889634f;
    const int c0 = part * 32;
    const float2 sc = make_float2(scale_log2, scale_log2);
    float* vec = sVec + (warp - 2) * 64;         // MODE 0: -lse*log2e and -D of this warp's 32 queries
    // Epilogue of the CTA's k-th item: accumulators -> dqkv (bf16).  The TMEM buffer is
    // released after the last read, before the global stores.
    auto epilogue = [&](const BwdItem& w, int k) -> bool {
      const int ab = (MODE == 0) ? 0 : (k & 1);
      if (!mbar_wait_warp(&acc_full[ab], (MODE == 0) ? (k & 1) : ((k >> 1) & 1), abort_flag)) return false;
      tc_fence_after();
      const int gi = w.tile * 128 + r;
      const int row0 = (w.bh / H) * T, h = w.bh % H;
      bf16* row = dqkv + (long long)(row0 + gi) * (3 * C) + h * HD + part * 16;
      // MODE 0: dV (column block 2C) and dK (column block C, times scale); MODE 1: dQ (times
      // scale).  Each of the 4 warps of a lane quarter writes 16 of the 64 head columns.
      constexpr int NA = (MODE == 0) ? 2 : 1;
      uint32_t u[NA][16];
#pragma unroll
      for (int a = 0; a < NA; ++a) tmem_ld16(tmem + lane_off + BACC_C + ab * 64 + a * 64 + part * 16, u[a]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      if (bias_part != nullptr) {
        const int b = w.bh / H;
        float* prow = bias_part + ((long long)(w.tile * B + b) * 4 + q) * (3 * C) + h * HD + part * 16 + (lane >> 1);
#pragma unroll
        for (int a = 0; a < NA; ++a) {
          const float mul = (MODE == 0 && a == 0) ? 1.0f : scale;
          float x[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) x[j] = (gi < T) ? __uint_as_float(u[a][j]) * mul : 0.f;
          const float cs = warp_colsum16(x, lane);
          if ((lane & 1) == 0) prow[(MODE == 1) ? 0 : (a == 0 ? 2 * C : C)] = cs;
        }
      }
      if (gi < T) {
#pragma unroll
        for (int a = 0; a < NA; ++a) {
          const float mul = (MODE == 0 && a == 0) ? 1.0f : scale;
          bf16* dst = row + ((MODE == 1) ? 0 : (a == 0 ? 2 * C : C));
#pragma unroll
          for (int gq = 0; gq < 2; ++gq) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(u[a][gq * 8 + 0]) * mul, __uint_as_float(u[a][gq * 8 + 1]) * mul);
            v.y = pack_bf16x2(__uint_as_float(u[a][gq * 8 + 2]) * mul, __uint_as_float(u[a][gq * 8 + 3]) * mul);
            v.z = pack_bf16x2(__uint_as_float(u[a][gq * 8 + 4]) * mul, __uint_as_float(u[a][gq * 8 + 5]) * mul);
            v.w = pack_bf16x2(__uint_as_float(u[a][gq * 8 + 6]) * mul, __uint_as_float(u[a][gq * 8 + 7]) * mul);
            reinterpret_cast<uint4*>(dst)[gq] = v;
          }
        }
      }
      return true;
    };
    bool ok = true;
    int g = 0;
    BwdItem prev{};
    int k = 0;
    for (;; ++k) {
      const int idx = bwd_turn_item(k);
      if (idx >= n_items) break;
      const BwdItem w = bwd_item<MODE>(idx, BH, n_t);
      const float* lse_bh = lse + (long long)w.bh * T;
      const float* D_bh = Dbuf + (long long)w.bh * T;
      // MODE 1: this thread's query row; a row past T gets P = 0 (its lse taken as +inf)
      float nl1 = 0.f, nd1 = 0.f;
      if (MODE == 1) {
        const int qi = w.tile * 128 + r;
        nl1 = (qi < T) ? -__ldg(lse_bh + qi) * LOG2E : -INFINITY;
        nd1 = (qi < T) ? -__ldg(D_bh + qi) : 0.f;
      }
      for (int t = w.it0; t < w.it1; ++t, ++g) {
        // MODE 0: the 32 queries of this warp's columns.  Lane i loads query t*128 + c0 + i's
        // scalars (a query past T gets P = 0) before the wait for the scores, stages them after
        // it (so the load latency hides behind the wait), and every lane then reads all 32.
        float nl0 = 0.f, nd0 = 0.f;
        if (MODE == 0) {
          const int qi = t * 128 + c0 + lane;
          nl0 = (qi < T) ? -__ldg(lse_bh + qi) * LOG2E : -INFINITY;
          nd0 = (qi < T) ? -__ldg(D_bh + qi) : 0.f;
        }
        if (!mbar_wait_warp(sd_full, g & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (MODE == 0) {
          __syncwarp();                            // the previous tile's reads of vec are done
          vec[lane] = nl0;
          vec[32 + lane] = nd0;
          __syncwarp();
        }
        // causal mask on the diagonal tile: MODE 0 drops queries before key r, MODE 1 keys after
        // query r.  There a warp's whole 32 x 32 chunk is masked when its columns all lie on the
        // masked side of its 32 rows (MODE 0: part < q; MODE 1: part > q): its P and dZ are zero
        // and its scores need no exponentials.
        const bool diag = (t == w.tile);
        const bool all_masked = diag && ((MODE == 0) ? (part < q) : (part > q));
        // The thread's 32 columns: all of S and the first 16 of dP come from TMEM first, and S
        // is released at once; dP's second half is read (and released) after the first half's
        // P and dZ are computed and stored.  Holding 64 of the 96 registers at most.
        auto pairs = [&](auto diag_tag, const uint32_t (&us)[32], const uint32_t (&ud)[16], int hf, uint32_t (&pw)[8],
                         uint32_t (&dw)[8]) {
          // P and dZ of 16 columns, with the causal mask only on the diagonal tile: the two
          // cases are separate code, so the other tiles carry no mask arithmetic
          constexpr bool DG = decltype(diag_tag)::value;
#pragma unroll
          for (int d = 0; d < 16; d += 4) {
            float4 nl4, nd4;   // the scalars of the 4 columns d .. d + 3
            if (MODE == 0) {
              nl4 = *reinterpret_cast<const float4*>(vec + 16 * hf + d);
              nd4 = *reinterpret_cast<const float4*>(vec + 32 + 16 * hf + d);
            } else {
              nl4 = make_float4(nl1, nl1, nl1, nl1);
              nd4 = make_float4(nd1, nd1, nd1, nd1);
            }
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int j = d + e;
              const float2 nl = e ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
              const float2 nd = e ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
              const float2 x = ffma2(make_float2(__uint_as_float(us[16 * hf + j]), __uint_as_float(us[16 * hf + j + 1])),
                                     sc, nl);
              float2 pp;
              if constexpr (DG) {
                const int c = c0 + 16 * hf + j;
                pp = all_masked ? make_float2(0.f, 0.f) : make_float2(ex2(x.x), ex2(x.y));
                if (MODE == 0) {
                  if (c < r) pp.x = 0.f;
                  if (c + 1 < r) pp.y = 0.f;
                } else {
                  if (c > r) pp.x = 0.f;
                  if (c + 1 > r) pp.y = 0.f;
                }
              } else {
                pp = make_float2(ex2(x.x), ex2(x.y));
              }
              const float2 gz = fmul2(pp, fadd2(make_float2(__uint_as_float(ud[j]), __uint_as_float(ud[j + 1])), nd));
              pw[j >> 1] = pack_bf16x2(pp.x, pp.y);
              dw[j >> 1] = pack_bf16x2(gz.x, gz.y);
            }
          }
        };
        uint32_t us[32], ud[16], pw[8], dw[8];
        tmem_ld32(tmem + lane_off + BS_C + c0, us);
        tmem_ld16(tmem + lane_off + BDP_C + c0, ud);
        tmem_wait_ld_regs(us);
        tmem_wait_ld_regs16(ud);
        tc_fence_before();
        mbar_arrive(s_empty);
        if (diag) pairs(std::true_type{}, us, ud, 0, pw, dw);
        else pairs(std::false_type{}, us, ud, 0, pw, dw);
        // the previous tile's MMAs must be done reading P / dZ in TMEM
        if (!mbar_wait_warp(ps_empty, (g & 1) ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (MODE == 0) tmem_st8(tmem + lane_off + BP_C + (c0 >> 1), pw);
        tmem_st8(tmem + lane_off + BDS_C + (c0 >> 1), dw);
        tmem_ld16(tmem + lane_off + BDP_C + c0 + 16, ud);
        tmem_wait_ld_regs16(ud);
        tc_fence_before();
        mbar_arrive(dp_empty);
        if (diag) pairs(std::true_type{}, us, ud, 1, pw, dw);
        else pairs(std::false_type{}, us, ud, 1, pw, dw);
        if (MODE == 0) tmem_st8(tmem + lane_off + BP_C + (c0 >> 1) + 8, pw);
        tmem_st8(tmem + lane_off + BDS_C + (c0 >> 1) + 8, dw);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ps_full);
        // the previous item's epilogue runs once this item's first tile is handed over, so
        // its wait for the last accumulation overlaps this item's products
        if (t == w.it0 && k > 0 && !epilogue(prev, k - 1)) { ok = false; break; }
      }
      if (!ok) break;
      prev = w;
    }
    if (ok && k > 0) epilogue(prev, k - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

int encode_rows64(CUtensorMap* tm, const void* base, int cols, long long rows) {
  PFN_encode fn = encode_fn();
  if (fn == nullptr) return -3;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return -1;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS ? 0 : -3;
}

}  // namespace

// Tensor-core backward for head size 64 in bf16 (D = rowsum(dO * O) precomputed).
int launch_attn_bwd_tc(cudaStream_t st, const void* qkv, const void* dout, const float* lse, const float* Dbuf,
                       void* dqkv, int B, int T, int H, int hd, float* bias_part) {
  if (hd != HD) return -4;
  if ((reinterpret_cast<uintptr_t>(dqkv) & 15) != 0) return -1;   // 16-byte stores of dQ, dK, dV
  const int C = H * HD;
  CUtensorMap tq, td;
  int rc = encode_rows64(&tq, qkv, 3 * C, (long long)B * T);
  if (rc) return rc;
  rc = encode_rows64(&td, dout, C, (long long)B * T);
  if (rc) return rc;
  const int nsm = current_device_sms();
  const int items = cdiv(T, 128) * B * H;
  const int grid = items < nsm ? items : nsm;   // persistent: one CTA per SM
  const float scale = 1.0f / sqrtf((float)HD);
  const float scale_log2 = 1.4426950408889634f * scale;
  if (set_dynamic_smem_once((const void*)attn_bwd_tc_kernel<0>, BWD_SMEM) ||
      set_dynamic_smem_once((const void*)attn_bwd_tc_kernel<1>, BWD_SMEM))
    return -3;
  attn_bwd_tc_kernel<0><<<grid, BWD_THREADS, BWD_SMEM, st>>>(tq, td, lse, Dbuf, reinterpret_cast<bf16*>(dqkv),
                                                             bias_part, B, T, H, scale, scale_log2);
  attn_bwd_tc_kernel<1><<<grid, BWD_THREADS, BWD_SMEM, st>>>(tq, td, lse, Dbuf, reinterpret_cast<bf16*>(dqkv),
                                                             bias_part, B, T, H, scale, scale_log2);
  if (rc) return rc;
  note_kernel_launches(2);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
