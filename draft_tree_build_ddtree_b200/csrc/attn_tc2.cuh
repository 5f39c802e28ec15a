// Stage 3, long key ranges: ancestor-only GQA tree attention with two M-tiles
// per CTA sharing every K/V tile, and P kept in tensor memory.
//
// "DDTree Deep Dive" §4 (a tree node attends to the committed prefix, the
// root, its ancestors and itself).  Same rows, mask and arithmetic as
// tree_attn_tc_kernel; what differs is how the work meets the hardware.
//
// Why: at full tensor-core rate the single-M-tile kernel would move about
// 250 bytes per clock through each SM's shared memory (the TMA writes of
// every K/V tile per 128 rows, the Q operand re-read by every QK^T step, P
// written by the softmax and read back by the PV product), against the
// roughly 128 bytes per clock that shared memory serves.  Here:
//   * two M-tiles (256 rows) per CTA share each 128-key K/V tile, halving
//     the TMA traffic per flop;
//   * QK^T runs at N = 128 keys (one A and one B operand of 4 KB per K=16
//     step and 64 clocks of tensor work);
//   * P is written by the softmax into tensor memory over its own S columns
//     and read from there as the A operand of O += P V (tcgen05.mma with A in
//     TMEM), so P never touches shared memory.
// That is about 125 bytes per clock per SM at full rate.
//
// Tensor memory (512 columns): S0|P0 [0,128), S1|P1 [128,256), O0 [256,384),
// O1 [384,512).  P(j) of M-tile t is stored as packed bf16 pairs in the first
// 64 columns of S_t: column c of a lane holds keys 2c and 2c+1 of that row.
//
// Warps (320 threads): 0-3 softmax of M-tile 0, 4-7 softmax of M-tile 1 (a
// thread owns one row = one TMEM lane), 8 the TMA producer, 9 TMEM
// allocation and the single-thread MMA issuer.  The MMA issue order per key
// tile j is PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): the tensor pipe computes one
// M-tile's products while the other M-tile's softmax runs.  tcgen05
// operations issued by one thread complete in issue order, so
//   * S_t(j+1) overwriting P_t(j) runs after PV_t(j) has read it, and
//   * when a softmax sees S_t(j) complete, PV_t(j-1) has completed too: the
//     softmax may then rescale O_t in place (no product is writing it).
// O is rescaled only when the running max grows by more than 2^8, as in the
// single-tile kernel.  Every mbarrier wait is bounded; on timeout the kernel
// flags DDTREE_STATUS_TIMEOUT, every role leaves its loop, waits (bounded)
// for its copies and products in flight and frees the tensor memory.  No TMA
// multicast is used.
#pragma once

#include <type_traits>

#include "attn_tc.cuh"
#include "exp2_poly.h"

namespace ddt {

constexpr int T2_THREADS = 320;
constexpr int T2_BN = 128;                          // keys per tile
constexpr int T2_KATOM = T2_BN * 64 * 2;            // [128 keys][64 dims] bf16: 16 KB
constexpr int T2_STAGES = 2;
constexpr uint32_t T2_TMEM_COLS = 512;
#ifndef T2_POLY
#define T2_POLY 0   // exponentials per eight on the FMA pipe (unmasked tiles)
#endif

// Head dim D in {64, 128}: a Q tile is D/64 swizzle atoms of [128 rows][64
// dims] (16 KB each), a K or V tile D/64 atoms of [128 keys][64 dims].
template <int D>
struct T2Smem {
  static constexpr int QTILE = (D / 64) * TC_ATOM;
  static constexpr int KTILE = (D / 64) * T2_KATOM;
  unsigned char q[2][QTILE];
  unsigned char k[T2_STAGES][KTILE];
  unsigned char v[T2_STAGES][KTILE];
  uint64_t bar_q, bar_kf[T2_STAGES], bar_ke[T2_STAGES], bar_vf[T2_STAGES], bar_ve[T2_STAGES];
  uint64_t bar_sfull[2], bar_pready[2], bar_odone;
  uint32_t tmem_base;
  int abort;
  int lpt_r;
};

template <int D>
constexpr size_t t2_smem_bytes() { return sizeof(T2Smem<D>); }


// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: two independent lanes, each
// rounded as the scalar operation would be).
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// max of three (sm_100 three-input max)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the FMA pipe, for x <= 2^8 with no -inf (unmasked keys): x is split
// into the nearest integer j (the 1.5*2^23 shifter, whose low bits then hold
// j) and f in [-1/2, 1/2]; 2^f is a degree-3 least-squares polynomial
// (coefficients from gen_exp2_poly.py; relative error 1.4e-4, below bf16's
// 2^-9 rounding of P) and j is added to the exponent field.  Inputs below
// -126 are clamped there (2^-126: a P that rounds to nothing against the row).
__device__ __forceinline__ float ex2_fma(float x) {
  x = fmaxf(x, -126.0f);
  const float r = __fadd_rn(x, 12582912.0f);
  const float f = __fsub_rn(x, __fsub_rn(r, 12582912.0f));
  float p = fmaf(EX2_POLY_C3, f, EX2_POLY_C2);
  p = fmaf(p, f, EX2_POLY_C1);
  p = fmaf(p, f, EX2_POLY_C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(r) << 23));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct T2Params {
  AttnGeom g;
  int G;               // query heads per KV head
  int mtiles;          // M-tiles per (layer, request, KV head)
  int mpairs;          // CTAs' M-tile groups per (layer, request, KV head): ceil(mtiles / nq)
  int nq;              // M-tiles per CTA (1 or 2)
  int splits;
  int units;           // layers * n_req * Hkv * mpairs
  const int32_t* block_table;
  const int32_t* prefix_len;
  const uint32_t* anc;
  const int32_t* n_nodes;
  __nv_bfloat16* out;
  float* out_lse;
  float* ws_o;         // partials per (M-tile unit, split), as for the combine kernel
  float2* ws_ml;
  int lpt;
  uint64_t wait_ns;
  int stop_tile;
  int early;           // 1: launched (EARLY instance) while the tree is still being built
};

// EARLY: the instance a round launches for a split key range directly after
// the build (see the host side); the plain instance reads the tree at once.
template <int D, bool EARLY>
__global__ void __launch_bounds__(T2_THREADS, 1)
tree_attn_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const T2Params p) {
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  typedef T2Smem<D> Smem;
  Smem& sm = *reinterpret_cast<Smem*>(smem_dyn);
  constexpr int HA = D / 64;                          // 64-dim atoms per row
  if ((smem_u32(smem_dyn) & 1023u) != 0u) {       // the 128B-swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) flag_status(DDTREE_STATUS_SETUP);
    return;
  }
  const AttnGeom& g = p.g;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // ---- which unit ----
  // The units of one (layer, request, KV head) are adjacent in launch order,
  // so they run close together in time and share its K/V through L2.
  const int split = blockIdx.x % p.splits;
  int u = blockIdx.x / p.splits;
  const int mp = u % p.mpairs;
  u /= p.mpairs;
  const int kvh = u % g.Hkv; u /= g.Hkv;
  int r = u % g.n_req; u /= g.n_req;
  const int layer = u;
  if (p.lpt) {     // ragged batch: longest key range first (see tree_attn_tc_kernel)
    const int r_slot = r;
    for (int i = tid; i < g.n_req; i += T2_THREADS) {
      const int ki = p.prefix_len[i] + p.n_nodes[i];
      int rank = 0;
      for (int j = 0; j < g.n_req; ++j) {
        const int kj = p.prefix_len[j] + p.n_nodes[j];
        rank += (kj > ki) || (kj == ki && j < i);
      }
      if (rank == r_slot) sm.lpt_r = i;
    }
    __syncthreads();
    r = sm.lpt_r;
  }
  const int nodes_per_tile = TC_BM / p.G;
  const int mt0 = mp * p.nq;                          // first M-tile of this CTA
  // EARLY: the build of this round's tree may still be running.  The CTA
  // tiles over the budget's node bound g.n (keys >= P + n_nodes are masked
  // anyway); its softmax warps wait for the build before their first tile if
  // the CTA's key range reaches the tree slots, else before the epilogue, the
  // only readers of the tree, so splits holding prefix tiles only run while
  // the tree is built.  Without room in the tiling (P + g.n beyond the
  // cache) it waits here.
  bool early = false;
  int nn;
  if constexpr (EARLY) {
    const int Pe = p.prefix_len[r];
    const long long cape = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
    early = p.early && Pe >= 0 && (long long)Pe + g.n <= cape;
    if (!early) griddep_wait();
    nn = early ? g.n : p.n_nodes[r];
  } else {
    nn = p.n_nodes[r];
  }
  const int node_base = mt0 * nodes_per_tile;
  if (node_base >= nn) return;                        // no live node in this CTA's M-tiles
  // M-tiles of this CTA holding a live node (1 or 2)
  const int ntl = (p.nq == 2 && node_base + nodes_per_tile < nn && mt0 + 1 < p.mtiles) ? 2 : 1;
  const int P = p.prefix_len[r];
  const long long cap = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
  if (P < 0 || (long long)P + nn > cap) {
    if (tid == 0 && mp == 0 && kvh == 0 && split == 0) flag_status(DDTREE_STATUS_CAPACITY);
    return;
  }
  if (g.paged) {
    const int nb = (P + nn + DDTREE_PAGE - 1) / DDTREE_PAGE;
    int bad = 0;
    for (int b = tid; b < nb; b += T2_THREADS) {
      const int blk = p.block_table[(size_t)r * g.max_blocks + b];
      bad |= (blk < 0 || blk >= g.num_blocks);
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0 && mp == 0 && kvh == 0 && split == 0) flag_status(DDTREE_STATUS_CAPACITY);
      return;
    }
  }
  const int T = P + nn;
  const int ntiles = (T + T2_BN - 1) / T2_BN;
  const int per = (ntiles + p.splits - 1) / p.splits;
  const int t_begin = split * per;
  const int t_end = min(ntiles, t_begin + per);
  const int nt = max(0, t_end - t_begin);

  if (tid == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < T2_STAGES; ++s) {
      mbar_init(&sm.bar_kf[s], 1);
      mbar_init(&sm.bar_ke[s], 1);
      mbar_init(&sm.bar_vf[s], 1);
      mbar_init(&sm.bar_ve[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.bar_sfull[t], 1);
      mbar_init(&sm.bar_pready[t], 128);
    }
    mbar_init(&sm.bar_odone, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "r"(T2_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  const float sl2 = g.scale * 1.4426950408889634f;   // scale * log2(e)
  const uint64_t wlim = p.wait_ns;

  if (warp == 8) {
    // =========================== TMA producer ===========================
    if (lane == 0 && nt > 0) {
      const int qb = layer * g.n_req + r;
      mbar_expect_tx(&sm.bar_q, (uint32_t)(ntl * Smem::QTILE));
      for (int t = 0; t < ntl; ++t) {
        const int nd = node_base + t * nodes_per_tile;
        for (int h = 0; h < HA; ++h)
          tma_load_4d(smem_u32(sm.q[t] + h * TC_ATOM), &tm_q, &sm.bar_q, 64 * h, kvh * p.G, nd, qb);
      }
      int issued = 0;
      for (int jj = 0; jj < nt; ++jj) {
        if (jj == p.stop_tile) break;      // diagnostics: withhold the rest, a consumer wait runs out
        const int j = t_begin + jj;
        const int st = jj % T2_STAGES;
        const int use = jj / T2_STAGES;
        const int k0 = j * T2_BN;
        int b0 = 0, b1 = 0;
        if (g.paged) {     // the tile's two pages; a second page past the validated range reuses the first (masked)
          const int pg = k0 / DDTREE_PAGE;
          const int maxpg = (T + DDTREE_PAGE - 1) / DDTREE_PAGE;
          b0 = p.block_table[(size_t)r * g.max_blocks + pg];
          b1 = (pg + 1 < maxpg) ? p.block_table[(size_t)r * g.max_blocks + pg + 1] : b0;
        }
        auto load_tile = [&](const CUtensorMap* map, unsigned char* tile, uint64_t* bar) {
          mbar_expect_tx(bar, Smem::KTILE);
          for (int h = 0; h < HA; ++h) {
            const uint32_t dst = smem_u32(tile + h * T2_KATOM);
            if (!g.paged) {
              tma_load_4d(dst, map, bar, 64 * h, kvh, k0, layer * g.n_req + r);
            } else {
              tma_load_4d(dst, map, bar, 64 * h, kvh, 0, layer * g.num_blocks + b0);
              tma_load_4d(dst + T2_KATOM / 2, map, bar, 64 * h, kvh, 0, layer * g.num_blocks + b1);
            }
          }
        };
        if (use > 0 && !mbar_wait(&sm.bar_ke[st], (use - 1) & 1, abort, wlim)) break;
        load_tile(&tm_k, sm.k[st], &sm.bar_kf[st]);
        if (use > 0 && !mbar_wait(&sm.bar_ve[st], (use - 1) & 1, abort, wlim)) break;
        load_tile(&tm_v, sm.v[st], &sm.bar_vf[st]);
        issued = jj + 1;
      }
      if (*abort || issued < nt) {       // copies in flight must land before the CTA exits
        int z = 0;
        mbar_wait(&sm.bar_q, 0, (volatile int*)&z);
        for (int jj = max(0, issued - T2_STAGES); jj < issued; ++jj) {
          mbar_wait(&sm.bar_kf[jj % T2_STAGES], (jj / T2_STAGES) & 1, (volatile int*)&z);
          mbar_wait(&sm.bar_vf[jj % T2_STAGES], (jj / T2_STAGES) & 1, (volatile int*)&z);
        }
      }
    }
  } else if (warp == 9) {
    // =========================== MMA issuer ===========================
    if (lane == 0 && nt > 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(TC_BM, T2_BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(TC_BM, D, false, true);
      bool ok = mbar_wait(&sm.bar_q, 0, abort, wlim);
      bool any_commit = false;
      // descriptors advance by (byte offset >> 4) in their 14-bit address field
      const uint64_t qd0 = smem_desc_sw128(smem_u32(sm.q[0]), 16, 1024);
      const uint64_t kd0 = smem_desc_sw128(smem_u32(sm.k[0]), 16, 1024);
      const uint64_t vd0 = smem_desc_sw128(smem_u32(sm.v[0]), T2_KATOM, 1024);
      auto issue_s = [&](int t, int st) {      // S_t = Q_t K^T over the 128 head dims
        const uint64_t qd = qd0 + (uint64_t)((t * Smem::QTILE) >> 4);
        const uint64_t kd = kd0 + (uint64_t)((st * Smem::KTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16(tmem + 128 * t, qd + (uint64_t)(((kk >> 2) * TC_ATOM + (kk & 3) * 32) >> 4),
                   kd + (uint64_t)(((kk >> 2) * T2_KATOM + (kk & 3) * 32) >> 4), IDESC_QK, kk > 0);
        umma_commit(&sm.bar_sfull[t]);
      };
      auto issue_pv = [&](int t, int st, int jj) {   // O_t += P_t V over the 128 keys
        const uint64_t vd = vd0 + (uint64_t)((st * Smem::KTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < T2_BN / 16; ++kk)
          umma_f16_ts(tmem + 256 + 128 * t, tmem + 128 * t + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), IDESC_PV,
                      (jj > 0 || kk > 0));
      };
      if (ok && mbar_wait(&sm.bar_kf[0], 0, abort, wlim)) {
        tc_fence_after();
        for (int t = 0; t < ntl; ++t) issue_s(t, 0);
        umma_commit(&sm.bar_ke[0]);
        any_commit = true;
      } else {
        ok = false;
      }
      for (int jj = 0; ok && jj < nt; ++jj) {
        const int st = jj % T2_STAGES;
        const int st1 = (jj + 1) % T2_STAGES;
        const bool more = jj + 1 < nt;
        if (!mbar_wait(&sm.bar_vf[st], (jj / T2_STAGES) & 1, abort, wlim)) break;
        bool kready = false;
        for (int t = 0; t < ntl; ++t) {
          if (!mbar_wait(&sm.bar_pready[t], jj & 1, abort, wlim)) { ok = false; break; }
          tc_fence_after();
          issue_pv(t, st, jj);
          if (more) {
            if (!kready) {
              if (!mbar_wait(&sm.bar_kf[st1], ((jj + 1) / T2_STAGES) & 1, abort, wlim)) { ok = false; break; }
              tc_fence_after();
              kready = true;
            }
            issue_s(t, st1);
          }
        }
        if (!ok) break;
        umma_commit(&sm.bar_ve[st]);
        if (more) umma_commit(&sm.bar_ke[st1]);
      }
      if (ok) {
        umma_commit(&sm.bar_odone);
      } else if (any_commit) {
        // products in flight must retire before the tensor memory is freed:
        // a commit to a fresh phase of O-done tracks every earlier product
        umma_commit(&sm.bar_odone);
        int z = 0;
        mbar_wait(&sm.bar_odone, 0, (volatile int*)&z);
      }
    }
  } else {
    // =========================== softmax warps ===========================
    const int t = warp >> 2;                               // M-tile of this warpgroup
    const int row = tid & 127;                             // TMEM lane == M row
    const int node = node_base + t * nodes_per_tile + row / p.G;
    const int hq = kvh * p.G + row % p.G;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tm_s = tmem + 128 * t + lane_off;
    const uint32_t tm_o = tmem + 256 + 128 * t + lane_off;
    const uint32_t* arow = p.anc + ((size_t)r * g.n + min(node, g.n - 1)) * g.W;
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = t < ntl;
    int nn_r = nn;                                         // the request's node count once the tree is read
    [[maybe_unused]] bool tree_seen = !early;
    if constexpr (EARLY) {
      if (!tree_seen && (long long)t_end * T2_BN > P) {   // this key range reaches the tree slots
        griddep_wait();
        nn_r = p.n_nodes[r];
        tree_seen = true;
      }
    }
    for (int jj = 0; ok && jj < nt; ++jj) {
      const int k0 = (t_begin + jj) * T2_BN;
      // tcgen05.ld/st are warp-collective: every exit and branch around them is warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull[t], jj & 1, abort, wlim))) { ok = false; break; }
      tc_fence_after();
      float s[T2_BN];
#pragma unroll
      for (int c = 0; c < T2_BN / 32; ++c) tmem_ld32(tm_s + c * 32, s + 32 * c);
      tmem_wait_ld();
      if (k0 + T2_BN > P) {     // keys >= P are tree slots (visible iff an ancestor); keys >= T absent
#pragma unroll
        for (int w = 0; w < T2_BN / 32; ++w) {
          const int j0 = k0 + 32 * w - P;              // tree index of the word's first key
          uint32_t word;
          if (j0 <= -32) {
            word = 0xffffffffu;
          } else if (j0 < 0) {
            word = (node < nn_r ? (arow[0] << (-j0)) : 0u) | ((1u << (-j0)) - 1u);
          } else {
            const int wi = j0 >> 5, sh = j0 & 31;
            const uint32_t lo = (node < nn_r && wi < g.W) ? arow[wi] : 0u;
            const uint32_t hi = (node < nn_r && wi + 1 < g.W) ? arow[wi + 1] : 0u;
            word = __funnelshift_r(lo, hi, sh);
          }
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (!((word >> c) & 1u)) s[32 * w + c] = -INFINITY;
        }
      }
      // The running max m_used only moves when a tile's max exceeds it by more
      // than 2^8 (then every P <= 256), so the exponentials need not wait for
      // this tile's max: P = 2^(s*sl2 - m_used) is computed and stored while the
      // tile's max is taken in the same pass; a tile that does exceed it (rare
      // after the first) rescales O and recomputes its P from the registers.  A
      // row without a finite max yet takes its max first.
      auto tile_max = [&]() {
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < T2_BN; c += 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) mx4[e] = max3f(mx4[e], s[c + 2 * e], s[c + 2 * e + 1]);
        }
        return max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;
      };
      // P of this tile with the current m_used into S's first 64 columns, two
      // keys per packed f32x2 instruction for the scaling and the sums; on
      // tiles without masked keys NPOLY of every eight exponentials run as a
      // polynomial on the FMA pipe (ex2_fma) beside the ex2 unit.  Returns the
      // row sum; *tmax receives the tile's max (log2 units).
      auto exp_pass = [&](auto npoly, float* tmax) {
        constexpr int NPOLY = decltype(npoly)::value;
        const float mneg = (m_used == -INFINITY) ? 0.f : -m_used;
        const unsigned long long sl2x2 = f2_pack(sl2, sl2), m2 = f2_pack(mneg, mneg);
        unsigned long long acc[2] = {0ull, 0ull};
        float mx2[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {           // 32 keys -> 16 packed columns per store
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float s0 = s[32 * q4 + 2 * c], s1 = s[32 * q4 + 2 * c + 1];
            mx2[c & 1] = max3f(mx2[c & 1], s0, s1);
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s0, s1), sl2x2, m2), x0, x1);
            const bool p0 = NPOLY >= 1 && (c & 3) == 3, p1 = NPOLY >= 2 && (c & 3) == 3;
            const float e0 = p0 ? ex2_fma(x0) : ex2_approx(x0);
            const float e1 = p1 ? ex2_fma(x1) : ex2_approx(x1);
            acc[c & 1] = f2_add(acc[c & 1], f2_pack(e0, e1));
            pk[c] = pack_bf16x2(e0, e1);
          }
          tmem_st16(tm_s + 16 * q4, pk);
        }
        *tmax = fmaxf(mx2[0], mx2[1]) * sl2;
        float lo, hi;
        f2_unpack(f2_add(acc[0], acc[1]), lo, hi);
        return lo + hi;
      };
      // O *= corr (per row) and l *= corr; PV_t(jj-1) has completed (it precedes
      // S_t(jj)), so O_t is ours to rescale
      auto rescale_o = [&](float corr) {
        l *= corr;
        if (jj > 0) {
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {          // 16 columns at a time: S stays in registers
            uint32_t o[16];
            tmem_ld16(tm_o + c * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
            tmem_st16(tm_o + c * 16, o);
          }
          tmem_wait_st();
        }
      };
      if (__any_sync(0xffffffffu, m_used == -INFINITY)) {   // rows without a max yet: take it first
        const float m_tile = tile_max();
        const bool set = m_used == -INFINITY && m_tile > -INFINITY;
        if (set) m_used = m_tile;                     // O and l are still zero for such rows
      }
      float m_tile;
      float lt = (k0 + T2_BN <= P) ? exp_pass(std::integral_constant<int, T2_POLY>(), &m_tile)
                                   : exp_pass(std::integral_constant<int, 0>(), &m_tile);
      const bool grow = m_tile > m_used + TC_RESCALE_LOG2;
      if (__any_sync(0xffffffffu, grow)) {
        tmem_wait_st();                               // the first pass's P stores land before they are redone
        const float m_new = grow ? m_tile : m_used;
        rescale_o(grow ? ex2_approx(m_used - m_new) : 1.f);
        m_used = m_new;
        lt = exp_pass(std::integral_constant<int, 0>(), &m_tile);
      }
      l += lt;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_pready[t]);
    }
    // ---- epilogue ----
    if constexpr (EARLY) {
      if (!tree_seen) {
        griddep_wait();
        nn_r = p.n_nodes[r];
        tree_seen = true;
      }
    }
    bool fin = ok && nt > 0;
    if (fin) fin = mbar_wait(&sm.bar_odone, 0, abort, wlim);
    const int mt = mt0 + t;
    const size_t munit = (((size_t)layer * g.n_req + r) * g.Hkv + kvh) * p.mtiles + mt;
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const bool live = node < nn_r && DDT_IN_RANGE(node, 0, g.n);
      if (p.splits == 1) {
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        __nv_bfloat16* orow =
            p.out + ((((size_t)layer * g.n_req + r) * g.n + min(node, g.n - 1)) * g.Hq + hq) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tm_o + c * 32, o);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 q4;
              q4.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
              q4.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
              q4.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
              q4.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c * 32 + e) = q4;
            }
          }
        }
        if (live && p.out_lse)
          p.out_lse[(((size_t)layer * g.n_req + r) * g.n + node) * g.Hq + hq] =
              (m_used + log2f(l)) * 0.6931471805599453f;
      } else {
        const size_t slot = munit * p.splits + split;
        float4* wo = reinterpret_cast<float4*>(p.ws_o) + slot * (D / 4) * TC_BM + row;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tm_o + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            wo[(size_t)((c * 32 + e) / 4) * TC_BM] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        }
        p.ws_ml[slot * TC_BM + row] = make_float2(m_used, l);
      }
    } else if (p.splits > 1 && t < ntl) {
      const size_t slot = munit * p.splits + split;
      p.ws_ml[slot * TC_BM + row] = make_float2(-INFINITY, 0.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(T2_TMEM_COLS));
  }
}

// ---------------------------------------------------------------- host side
// Which kernel runs: the two-M-tile kernel whenever each CTA keeps at least
// T2_MIN_TILES key tiles after the split the GPU needs (long key ranges) and
// its CTAs still cover half the SMs; the single-M-tile kernel otherwise
// (short ranges, where set-up and latency dominate).
constexpr int T2_MIN_TILES = 8;

struct AttnDispatch {
  bool v2;
  TcPlan v1;           // single-M-tile plan (v2 == false)
  int splits, mtiles, mpairs, units2;   // two-M-tile plan
};

inline AttnDispatch attn_dispatch(const AttnGeom& g, int num_sms) {   // D = 64: always the two-M-tile kernel
  AttnDispatch d;
  d.v1 = tc_plan(g, num_sms);
  const int G = g.Hq / g.Hkv;
  d.mtiles = (g.n * G + TC_BM - 1) / TC_BM;
  d.mpairs = (d.mtiles + 1) / 2;
  d.units2 = g.layers * g.n_req * g.Hkv * d.mpairs;
  const long long cap = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
  const long long tiles = (cap + T2_BN - 1) / T2_BN;
  int splits = 1;
  if (d.units2 < num_sms) {
    splits = num_sms / d.units2;
    if (splits > TC_MAX_SPLITS) splits = TC_MAX_SPLITS;
    if ((long long)splits * T2_MIN_TILES > tiles) splits = (int)(tiles / T2_MIN_TILES);
    if (splits < 1) splits = 1;
  }
  d.splits = splits;
  // long enough per CTA, and enough CTAs to keep at least half the SMs busy;
  // the single-M-tile kernel is built for D = 128 only
  d.v2 = g.D == 64 || (tiles / splits >= T2_MIN_TILES && (long long)d.units2 * splits * 2 >= num_sms);
  return d;
}

inline size_t attn_tc_ws_bytes(const AttnGeom& g, int num_sms) {
  const AttnDispatch d = attn_dispatch(g, num_sms);
  if (!d.v2) return tc_attn_ws_bytes(g, num_sms);
  if (d.splits == 1) return 0;
  const size_t slots = (size_t)g.layers * g.n_req * g.Hkv * d.mtiles * d.splits;
  return align256(slots * TC_BM * g.D * 4) + align256(slots * TC_BM * 8);
}

inline int attn_tc_launch(const void* q, const void* kc, const void* vc, const int32_t* block_table,
                          const int32_t* prefix_len, const uint32_t* anc, const int32_t* n_nodes, const AttnGeom& g,
                          void* out, float* out_lse, void* ws, int num_sms, cudaStream_t stream,
                          uint64_t wait_ns = 0, int stop_tile = -1, int early = 0) {
  // early: inside a round, directly after the build.  The single-M-tile
  // kernel then starts while the tree is built; so does this kernel's EARLY
  // instance for a split key range.  Unsplit units reach the tree slots at
  // once, and the late wait costs the 168-register softmax spills, so they
  // take the plain instance and launch plainly.
  const AttnDispatch d = attn_dispatch(g, num_sms);
  if (!d.v2)
    return tc_attn_launch(q, kc, vc, block_table, prefix_len, anc, n_nodes, g, out, out_lse, ws, num_sms, stream,
                          wait_ns, stop_tile, early);
  T2Params p;
  p.g = g;
  p.G = g.Hq / g.Hkv;
  p.mtiles = d.mtiles;
  p.mpairs = d.mpairs;
  p.nq = 2;
  p.splits = d.splits;
  p.units = d.units2;
  p.block_table = block_table;
  p.prefix_len = prefix_len;
  p.anc = anc;
  p.n_nodes = n_nodes;
  p.out = (__nv_bfloat16*)out;
  p.out_lse = out_lse;
  p.ws_o = nullptr;
  p.ws_ml = nullptr;
  p.lpt = (d.splits == 1 && g.n_req > 1 && g.n_req <= TC_LPT_MAX_REQ) ? 1 : 0;
  p.wait_ns = wait_ns > 0 ? wait_ns : TC_WAIT_NS;
  p.stop_tile = stop_tile;
  p.early = (early && !g.paged && !p.lpt && d.splits > 1) ? 1 : 0;
  const size_t slots = (size_t)g.layers * g.n_req * g.Hkv * d.mtiles * d.splits;
  if (d.splits > 1) {
    p.ws_o = (float*)ws;
    p.ws_ml = (float2*)((char*)ws + align256(slots * TC_BM * g.D * 4));
  }
  CUtensorMap mq, mk, mv;
  const uint64_t D = (uint64_t)g.D;
  if (!make_map_4d(&mq, q, (uint64_t)g.Hq, (uint64_t)g.n, (uint64_t)g.layers * g.n_req, (uint32_t)p.G,
                   (uint32_t)(TC_BM / p.G), D))
    return cuda_fail_msg("tree attention: tensor map of q");
  if (!g.paged) {
    if (!make_map_4d(&mk, kc, g.Hkv, g.s_max, (uint64_t)g.layers * g.n_req, 1, T2_BN, D) ||
        !make_map_4d(&mv, vc, g.Hkv, g.s_max, (uint64_t)g.layers * g.n_req, 1, T2_BN, D))
      return cuda_fail_msg("tree attention: tensor map of the cache");
  } else {
    if (!make_map_4d(&mk, kc, g.Hkv, DDTREE_PAGE, (uint64_t)g.layers * g.num_blocks, 1, DDTREE_PAGE, D) ||
        !make_map_4d(&mv, vc, g.Hkv, DDTREE_PAGE, (uint64_t)g.layers * g.num_blocks, 1, DDTREE_PAGE, D))
      return cuda_fail_msg("tree attention: tensor map of the paged cache");
  }
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(tree_attn_tc2_kernel<128, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)t2_smem_bytes<128>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_attn_tc2_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)t2_smem_bytes<64>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_attn_tc2_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)t2_smem_bytes<128>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_attn_tc2_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)t2_smem_bytes<64>());
    if (e != cudaSuccess) return cuda_fail(e, "tree attention (two M-tiles): shared-memory attribute");
    attr_set = true;
  }
  const long long grid = (long long)d.units2 * d.splits;
  if (grid > 0x7fffffffLL) return DDTREE_ERR_UNSUPPORTED;
  {
    const dim3 gd((unsigned)grid), bd(T2_THREADS);
    cudaError_t e;
    if (p.early)
      e = g.D == 64 ? launch_maybe_pdl(tree_attn_tc2_kernel<64, true>, gd, bd, t2_smem_bytes<64>(), stream, true, mq,
                                       mk, mv, p)
                    : launch_maybe_pdl(tree_attn_tc2_kernel<128, true>, gd, bd, t2_smem_bytes<128>(), stream, true,
                                       mq, mk, mv, p);
    else if (g.D == 64)
      tree_attn_tc2_kernel<64, false><<<gd, bd, t2_smem_bytes<64>(), stream>>>(mq, mk, mv, p);
    else
      tree_attn_tc2_kernel<128, false><<<gd, bd, t2_smem_bytes<128>(), stream>>>(mq, mk, mv, p);
    if (!p.early || e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "tree attention (two M-tiles): launch");
  }
  if (d.splits > 1) {
    // the combine kernel walks M-tile units
    TcParams c;
    c.g = g;
    c.G = p.G;
    c.mtiles = d.mtiles;
    c.splits = d.splits;
    c.units = g.layers * g.n_req * g.Hkv * d.mtiles;
    c.block_table = block_table;
    c.prefix_len = prefix_len;
    c.anc = anc;
    c.n_nodes = n_nodes;
    c.out = p.out;
    c.out_lse = out_lse;
    c.ws_o = p.ws_o;
    c.ws_ml = p.ws_ml;
    c.lpt = 0;
    c.wait_ns = p.wait_ns;
    c.stop_tile = -1;
    c.early = 0;
    const unsigned cgrid = (unsigned)(c.units * (g.D / 8));
    if (g.D == 64) {
      if (d.splits <= 8) tree_attn_combine_kernel<8, 64><<<cgrid, TC_BM, 0, stream>>>(c);
      else tree_attn_combine_kernel<TC_MAX_SPLITS, 64><<<cgrid, TC_BM, 0, stream>>>(c);
    } else {
      if (d.splits <= 8) tree_attn_combine_kernel<8><<<cgrid, TC_BM, 0, stream>>>(c);
      else tree_attn_combine_kernel<TC_MAX_SPLITS><<<cgrid, TC_BM, 0, stream>>>(c);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "tree attention: combine launch");
  }
  return DDTREE_OK;
}

}  // namespace ddt
