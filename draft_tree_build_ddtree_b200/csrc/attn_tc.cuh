// Stage 3 (tensor-core path): ancestor-only GQA tree attention on sm_100a.
//
// "DDTree Deep Dive" §4: every tree node attends to the committed prefix
// (KV cache), the root, its ancestors and itself, never to siblings or other
// branches.  The autobench DDTree page notes that this mask is why the pages'
// verifier falls back to a dense masked SDPA; here it is applied inside a
// flash-style kernel instead.
//
// Layout of the work.  The B+1 tree nodes times the G = Hq/Hkv query heads
// that share one KV head form a dense M dimension: an M-tile is 128 rows =
// (128/G nodes) x (G heads), row t = node_local*G + head_local, which TMA
// loads in one box from q[layer][req][node][head][D].  One CTA handles one
// (layer, request, KV head, M-tile, key split).
//
// Per key tile (64 or 128 keys, TcCfg):  S = Q K^T (tcgen05.mma kind::f16, A and B K-major from
// 128B-swizzled shared memory, fp32 accumulator in TMEM), then the softmax
// warps read S from TMEM (one thread per row = TMEM lane), apply the
// ancestor mask only on tiles that reach the tree slots, update the running
// max/sum, write P = exp2(S*scale*log2e - m) as packed bf16 pairs into
// tensor-memory columns of its own, and O += P V (tcgen05.mma with the A
// operand in TMEM, V as an MN-major operand from shared memory) accumulates
// in TMEM.  O is rescaled only when the running max grows by more than 2^8,
// which keeps every P <= 256 and leaves the final O / l exact.  K and V tiles
// are double buffered; S is released as soon as the softmax has loaded it,
// so the QK^T of the next tile overlaps the softmax of the current one.
// (P in tensor memory instead of shared memory: b64_p2k attention 15.1 vs
// 15.5 us, and 1.92 vs 2.05 ms when this kernel runs the 48-layer B = 256
// workload.)
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue (warp w reads TMEM
// lanes 32w..32w+31), warp 4 the TMA producer, warp 5 TMEM allocation and
// the single-thread MMA issue.  Every mbarrier wait is bounded (about one
// second by default); on timeout the kernel sets DDTREE_STATUS_TIMEOUT, every role
// leaves its loop, waits (bounded) for its copies and MMAs in flight, and
// the TMEM is freed before exit.  No TMA multicast is used.
//
// When the key range is split across CTAs, each split writes its unnormalised
// O, running max and sum to the workspace and a combine kernel merges them.
// Unsplit launches over a ragged batch take the requests longest key range
// first, so the longest units start in the first wave.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "attn_simt.cuh"

namespace ddt {

constexpr int TC_THREADS = 192;
constexpr int TC_BM = 128;        // rows per M-tile
constexpr int TC_D = 128;         // head dim
constexpr int TC_ATOM = TC_BM * 64 * 2;     // one [128][64] bf16 swizzle-128B atom column: 16 KB
constexpr int TC_TILE = 2 * TC_ATOM;        // [128][128] bf16: 32 KB (Q)
constexpr int TC_MIN_SPLIT_TILES = 4;
constexpr int TC_SHORT_TILES = 6;

// Key-tile variants: 128 keys per tile, one CTA per SM (short, split key
// ranges: fewer tiles per CTA), or 64 keys (one KV page) per tile, two CTAs
// per SM (long key ranges: the two CTAs' softmax and MMAs interleave).
template <int BN>
struct TcCfg {
  static constexpr int KATOM = BN * 64 * 2;     // one [BN keys][64 dims] bf16 atom
  static constexpr int KTILE = 2 * KATOM;       // a K or V tile [BN keys][128 dims]
  static constexpr int CTAS = BN == 64 ? 2 : 1; // CTAs per SM
  // tensor memory: S [0, BN), O [BN, BN+128), P [BN+128, BN+128+BN/2)
  // (bf16 pairs); 224 of 256 columns at BN = 64 (two CTAs per SM), 320 of 512
  // at BN = 128
  static constexpr uint32_t TMEM_COLS = BN == 64 ? 256 : 512;
};
constexpr int TC_STAGES = 2;
constexpr float TC_RESCALE_LOG2 = 8.0f;

inline bool tc_attn_supported(int group) { return group >= 1 && group <= TC_BM && (TC_BM % group) == 0; }

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

constexpr uint64_t TC_WAIT_NS = 1000000000ull;   // one second

// Bounded wait for the phase of parity `parity`; false on timeout (after
// limit_ns) or when another role already gave up (*abort set).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns = TC_WAIT_NS) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort = 1;
      flag_status(DDTREE_STATUS_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (16-byte units), version 1, 128B swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                 // descriptor version for tcgen05
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, M=128, N=128.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)   // A major
         | ((b_mn_major ? 1u : 0u) << 16)   // B major
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// D[tmem] (+)= A[tmem] * B[smem]: kind::f16 with the A operand in tensor memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- parameters
struct TcParams {
  AttnGeom g;
  int G;               // query heads per KV head
  int mtiles;          // M-tiles per (layer, request, KV head)
  int splits;          // key splits per M-tile
  int units;           // layers * n_req * Hkv * mtiles
  const int32_t* block_table;
  const int32_t* prefix_len;
  const uint32_t* anc;
  const int32_t* n_nodes;
  __nv_bfloat16* out;
  float* out_lse;
  float* ws_o;         // [units*splits][128][128] partial O (splits > 1)
  float2* ws_ml;       // [units*splits][128] (max in log2 units, sum)
  int lpt;             // 1: requests taken longest key range first (unsplit only)
  uint64_t wait_ns;    // limit of the pipeline's bounded waits
  int stop_tile;       // >= 0: the producer issues no key tile from this one on (timeout-path diagnostics)
  int early;           // 1: launched while the tree is still being built (see the kernel)
};

template <int BN>
struct TcSmem {
  // 1024-byte aligned tiles first
  unsigned char q[TC_TILE];
  unsigned char k[TC_STAGES][TcCfg<BN>::KTILE];
  unsigned char v[TC_STAGES][TcCfg<BN>::KTILE];
  uint64_t bar_q, bar_kf[TC_STAGES], bar_ke[TC_STAGES], bar_vf[TC_STAGES], bar_ve[TC_STAGES];
  uint64_t bar_sfull, bar_sfree, bar_pfull, bar_pvdone;
  uint32_t tmem_base;
  int abort;
  int blk[2];
  int lpt_r;
};

// Two CTAs share an SM, so there is no room for alignment slack: the
// dynamic shared memory (no static shared memory in the kernel) starts at
// shared address 0, which the kernel checks.
template <int BN>
constexpr size_t tc_smem_bytes() { return sizeof(TcSmem<BN>); }

// ---------------------------------------------------------------- the kernel
template <int BN>
__global__ void __launch_bounds__(TC_THREADS, TcCfg<BN>::CTAS)
tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const TcParams p) {
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  constexpr int TC_BN = BN;
  constexpr int TC_KATOM = TcCfg<BN>::KATOM;
  constexpr int TC_KTILE = TcCfg<BN>::KTILE;
  TcSmem<BN>& sm = *reinterpret_cast<TcSmem<BN>*>(smem_dyn);
  if ((smem_u32(smem_dyn) & 1023u) != 0u) {       // the 128B-swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) flag_status(DDTREE_STATUS_SETUP);
    return;
  }
  const AttnGeom& g = p.g;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // ---- which unit ----
  const int split = blockIdx.x % p.splits;
  int u = blockIdx.x / p.splits;
  const int unit = u;
  const int mt = u % p.mtiles; u /= p.mtiles;
  const int kvh = u % g.Hkv; u /= g.Hkv;
  int r = u % g.n_req; u /= g.n_req;
  const int layer = u;
  if (p.lpt) {
    // Ragged batch: request slot r takes the request of rank r in the order
    // of key count (prefix + nodes) descending, ties by index, so the
    // longest units are dispatched first and the last wave holds short ones.
    const int r_slot = r;
    for (int i = tid; i < g.n_req; i += TC_THREADS) {
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
  const int node0 = mt * nodes_per_tile;
  const int P = p.prefix_len[r];
  const long long cap = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
  // Early start (inside a round, contiguous cache): the build of this round's
  // tree may still be running.  The CTA tiles over the budget's node bound
  // g.n (keys >= P + n_nodes are masked anyway) and its softmax warps wait for
  // the build only before the first tile holding tree slots and before the
  // epilogue, which are the only readers of the tree.  Otherwise it waits here.
  const bool early = p.early && P >= 0 && (long long)P + g.n <= cap;
  if (!early) griddep_wait();
  const int nn = early ? g.n : p.n_nodes[r];     // node bound of the tiling
  if (node0 >= nn) return;                       // this M-tile holds no live node
  if (P < 0 || (long long)P + nn > cap) {
    if (tid == 0 && mt == 0 && kvh == 0 && split == 0) flag_status(DDTREE_STATUS_CAPACITY);
    return;
  }
  if (g.paged) {
    const int nb = (P + nn + DDTREE_PAGE - 1) / DDTREE_PAGE;
    int bad = 0;
    for (int b = tid; b < nb; b += TC_THREADS) {
      const int blk = p.block_table[(size_t)r * g.max_blocks + b];
      bad |= (blk < 0 || blk >= g.num_blocks);
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0 && mt == 0 && kvh == 0 && split == 0) flag_status(DDTREE_STATUS_CAPACITY);
      return;
    }
  }
  const int T = P + nn;                                   // keys of this request
  const int ntiles = (T + TC_BN - 1) / TC_BN;
  const int per = (ntiles + p.splits - 1) / p.splits;
  const int t_begin = split * per;
  const int t_end = min(ntiles, t_begin + per);
  const int nt = max(0, t_end - t_begin);

  if (tid == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&sm.bar_kf[s], 1);
      mbar_init(&sm.bar_ke[s], 1);
      mbar_init(&sm.bar_vf[s], 1);
      mbar_init(&sm.bar_ve[s], 1);
    }
    mbar_init(&sm.bar_sfull, 1);
    mbar_init(&sm.bar_sfree, 128);
    mbar_init(&sm.bar_pfull, 128);
    mbar_init(&sm.bar_pvdone, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "r"(TcCfg<BN>::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_s = tmem;              // cols [0, BN)
  const uint32_t tmem_o = tmem + TC_BN;      // cols [BN, BN+128)
  const uint32_t tmem_p = tmem + TC_BN + TC_D;   // cols [BN+128, BN+128+BN/2): P as bf16 pairs
  volatile int* abort = &sm.abort;
  const float sl2 = g.scale * 1.4426950408889634f;   // scale * log2(e)

  if (warp == 4) {
    // =========================== TMA producer ===========================
    if (lane == 0 && nt > 0) {
      const int qb = layer * g.n_req + r;
      mbar_expect_tx(&sm.bar_q, TC_TILE);
      tma_load_4d(smem_u32(sm.q), &tm_q, &sm.bar_q, 0, kvh * p.G, node0, qb);
      tma_load_4d(smem_u32(sm.q + TC_ATOM), &tm_q, &sm.bar_q, 64, kvh * p.G, node0, qb);
      int issued = 0;
      for (int jj = 0; jj < nt; ++jj) {
        if (jj == p.stop_tile) break;      // diagnostics: withhold the rest, a consumer wait runs out
        const int j = t_begin + jj;
        const int st = jj % TC_STAGES;
        const int use = jj / TC_STAGES;
        const int k0 = j * TC_BN;
        // KV pages of this tile (paged: their blocks through the block table; a
        // 128-key tile whose second page lies past the validated range reuses
        // the first, whose keys are masked)
        int b0 = 0, b1 = 0;
        if (g.paged) {
          const int pg = k0 / DDTREE_PAGE;
          const int maxpg = (T + DDTREE_PAGE - 1) / DDTREE_PAGE;   // validated blocks
          b0 = p.block_table[(size_t)r * g.max_blocks + pg];
          b1 = (BN > DDTREE_PAGE && pg + 1 < maxpg) ? p.block_table[(size_t)r * g.max_blocks + pg + 1] : b0;
        }
        auto load_tile = [&](const CUtensorMap* map, unsigned char* tile, uint64_t* bar) {
          mbar_expect_tx(bar, TC_KTILE);
          for (int h = 0; h < 2; ++h) {
            const uint32_t dst = smem_u32(tile + h * TC_KATOM);
            if (!g.paged) {
              tma_load_4d(dst, map, bar, 64 * h, kvh, k0, layer * g.n_req + r);
            } else {
              tma_load_4d(dst, map, bar, 64 * h, kvh, 0, layer * g.num_blocks + b0);
              if (BN > DDTREE_PAGE)
                tma_load_4d(dst + TC_KATOM / 2, map, bar, 64 * h, kvh, 0, layer * g.num_blocks + b1);
            }
          }
        };
        // K tile
        if (use > 0 && !mbar_wait(&sm.bar_ke[st], (use - 1) & 1, abort, p.wait_ns)) break;
        load_tile(&tm_k, sm.k[st], &sm.bar_kf[st]);
        // V tile
        if (use > 0 && !mbar_wait(&sm.bar_ve[st], (use - 1) & 1, abort, p.wait_ns)) break;
        load_tile(&tm_v, sm.v[st], &sm.bar_vf[st]);
        issued = jj + 1;
      }
      // copies in flight must land before the CTA exits
      if (*abort || issued < nt) {
        mbar_wait(&sm.bar_q, 0, abort);
        for (int jj = max(0, issued - TC_STAGES); jj < issued; ++jj) {
          int z = 0;
          mbar_wait(&sm.bar_kf[jj % TC_STAGES], (jj / TC_STAGES) & 1, (volatile int*)&z);
          mbar_wait(&sm.bar_vf[jj % TC_STAGES], (jj / TC_STAGES) & 1, (volatile int*)&z);
        }
      }
    }
  } else if (warp == 5) {
    // =========================== MMA issuer ===========================
    if (lane == 0 && nt > 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(TC_BM, TC_BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(TC_BM, TC_D, false, true);
      const uint32_t q_addr = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.bar_q, 0, abort, p.wait_ns);
      int committed_pv = 0, committed_qk = 0;
      for (int jj = 0; ok && jj <= nt; ++jj) {
        if (jj < nt) {
          const int st = jj % TC_STAGES;
          if (!mbar_wait(&sm.bar_kf[st], (jj / TC_STAGES) & 1, abort, p.wait_ns)) break;
          if (jj > 0 && !mbar_wait(&sm.bar_sfree, (jj - 1) & 1, abort, p.wait_ns)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm.k[st]);
#pragma unroll
          for (int kk = 0; kk < TC_D / 16; ++kk) {
            const uint32_t qoff = (kk >> 2) * TC_ATOM + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * TC_KATOM + (kk & 3) * 32;
            umma_f16(tmem_s, smem_desc_sw128(q_addr + qoff, 16, 1024), smem_desc_sw128(k_addr + koff, 16, 1024),
                     IDESC_QK, kk > 0);
          }
          umma_commit(&sm.bar_sfull);
          umma_commit(&sm.bar_ke[st]);
          committed_qk = jj + 1;
        }
        if (jj > 0) {
          const int pj = jj - 1;
          const int st = pj % TC_STAGES;
          if (!mbar_wait(&sm.bar_pfull, pj & 1, abort, p.wait_ns)) break;
          if (!mbar_wait(&sm.bar_vf[st], (pj / TC_STAGES) & 1, abort, p.wait_ns)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sm.v[st]);
#pragma unroll
          for (int kk = 0; kk < TC_BN / 16; ++kk)       // P from tensor memory: 16 keys = 8 columns per step
            umma_f16_ts(tmem_o, tmem_p + kk * 8, smem_desc_sw128(v_addr + kk * 16 * 128, TC_KATOM, 1024), IDESC_PV,
                        (pj > 0 || kk > 0));
          umma_commit(&sm.bar_pvdone);
          umma_commit(&sm.bar_ve[st]);
          committed_pv = jj;
        }
      }
      // MMAs in flight must retire before TMEM is freed
      if (*abort) {
        int z = 0;
        if (committed_qk > 0) mbar_wait(&sm.bar_sfull, (committed_qk - 1) & 1, (volatile int*)&z);
        if (committed_pv > 0) mbar_wait(&sm.bar_pvdone, (committed_pv - 1) & 1, (volatile int*)&z);
      }
    }
  } else {
    // =========================== softmax warps ===========================
    const int row = tid;                                  // TMEM lane == M row
    const int node = node0 + row / p.G;
    const int hq = kvh * p.G + row % p.G;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t* arow = p.anc + ((size_t)r * g.n + min(node, g.n - 1)) * g.W;
    // this row's node exists (1) or not (0); -1 until the build is seen done
    int row_live = early ? -1 : (node < nn ? 1 : 0);
    auto see_tree = [&]() {
      if (row_live < 0) {
        griddep_wait();
        row_live = node < p.n_nodes[r] ? 1 : 0;
      }
    };
    float m_used = -INFINITY;      // running max (log2 units) the accumulation uses
    float l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < nt; ++jj) {
      const int j = t_begin + jj;
      const int k0 = j * TC_BN;
      // tcgen05.ld/st are warp-collective: every exit and branch around them is warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_sfull, jj & 1, abort, p.wait_ns))) { ok = false; break; }
      tc_fence_after();
      float s[TC_BN];
#pragma unroll
      for (int c = 0; c < TC_BN / 32; ++c) tmem_ld32(tmem_s + lane_off + c * 32, s + 32 * c);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sm.bar_sfree);
      // mask: keys >= P are tree slots (visible iff an ancestor), keys >= T absent.
      // Four 32-key visibility words per tile, built from the node's ancestor row.
      if (k0 + TC_BN > P) {
        see_tree();
        uint32_t mw[TC_BN / 32];
#pragma unroll
        for (int w = 0; w < TC_BN / 32; ++w) {
          const int kb = k0 + 32 * w;
          const int j0 = kb - P;                       // tree index of the word's first key
          uint32_t word;
          if (j0 <= -32) {
            word = 0xffffffffu;                        // all prefix keys
          } else if (j0 < 0) {
            word = (row_live ? (arow[0] << (-j0)) : 0u) | ((1u << (-j0)) - 1u);
          } else {
            const int wi = j0 >> 5, sh = j0 & 31;
            const uint32_t lo = (row_live && wi < g.W) ? arow[wi] : 0u;
            const uint32_t hi = (row_live && wi + 1 < g.W) ? arow[wi + 1] : 0u;
            word = __funnelshift_r(lo, hi, sh);
          }
          mw[w] = word;
        }
#pragma unroll
        for (int c = 0; c < TC_BN; ++c)
          if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < TC_BN; c += 4) {
#pragma unroll
        for (int t = 0; t < 4; ++t) mx4[t] = fmaxf(mx4[t], s[c + t]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const float m_tile = mx * sl2;
      bool rescale = false;
      float m_new = m_used;
      if (m_tile > m_used + TC_RESCALE_LOG2 || (m_used == -INFINITY && m_tile > -INFINITY)) {
        m_new = m_tile;
        rescale = true;
      }
      // P = exp2(s*sl2 - m) as packed bf16 in registers first (exp2(-inf) = 0
      // masks), so the exponentials overlap the previous tile's PV product
      const float m_eff = rescale ? m_new : m_used;
      const float mneg = (m_eff == -INFINITY) ? 0.f : -m_eff;
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[TC_BN / 2];
#pragma unroll
      for (int ch = 0; ch < TC_BN / 8; ++ch) {       // 8 keys at a time
        float e[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) e[t] = exp2f(fmaf(s[ch * 8 + t], sl2, mneg));
#pragma unroll
        for (int t = 0; t < 4; ++t) pk[ch * 4 + t] = pack_bf16x2(e[2 * t], e[2 * t + 1]);
#pragma unroll
        for (int t = 0; t < 8; ++t) ls4[t & 3] += e[t];
      }
      // P buffer and O are free once the previous PV has retired
      if (jj > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_pvdone, (jj - 1) & 1, abort, p.wait_ns))) { ok = false; break; }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
        const float corr = !rescale ? 1.f : ((m_used == -INFINITY) ? 0.f : exp2f(m_used - m_new));
        l *= corr;
        if (jj > 0) {
#pragma unroll 1
          for (int c = 0; c < TC_D / 32; ++c) {
            float o[32];
            tmem_ld32(tmem_o + lane_off + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= corr;
            tmem_st32(tmem_o + lane_off + c * 32, o);
          }
          tmem_wait_st();
        }
        if (rescale) m_used = m_new;
      }
      l += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      // P into its tensor-memory columns (this thread's lane), the PV product's A operand
#pragma unroll
      for (int c = 0; c < TC_BN / 64; ++c) tmem_st32(tmem_p + lane_off + 32 * c, reinterpret_cast<const float*>(pk + 32 * c));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.bar_pfull);
    }
    // ---- epilogue ----
    see_tree();
    bool fin = ok && nt > 0;
    if (fin) fin = mbar_wait(&sm.bar_pvdone, (nt - 1) & 1, abort, p.wait_ns);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const bool live = row_live != 0;
      if (p.splits == 1) {
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        __nv_bfloat16* orow =
            p.out + ((((size_t)layer * g.n_req + r) * g.n + min(node, g.n - 1)) * g.Hq + hq) * TC_D;
#pragma unroll 1
        for (int c = 0; c < TC_D / 32; ++c) {
          float o[32];
          tmem_ld32(tmem_o + lane_off + c * 32, o);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 pk;
              pk.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
              pk.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
              pk.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
              pk.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c * 32 + e) = pk;
            }
          }
        }
        if (live && p.out_lse)
          p.out_lse[(((size_t)layer * g.n_req + r) * g.n + node) * g.Hq + hq] =
              (m_used + log2f(l)) * 0.6931471805599453f;
      } else {
        const size_t slot = (size_t)unit * p.splits + split;
        // [slot][D/4][128 rows] float4: a warp's 32 rows write 512 contiguous bytes per store
        float4* wo = reinterpret_cast<float4*>(p.ws_o) + slot * (TC_D / 4) * TC_BM + row;
#pragma unroll 1
        for (int c = 0; c < TC_D / 32; ++c) {
          float o[32];
          tmem_ld32(tmem_o + lane_off + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            wo[(size_t)((c * 32 + e) / 4) * TC_BM] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        }
        p.ws_ml[slot * TC_BM + row] = make_float2(m_used, l);
      }
    } else if (p.splits > 1) {
      // an empty (or aborted) split contributes nothing to the combine
      const size_t slot = (size_t)unit * p.splits + split;
      p.ws_ml[slot * TC_BM + row] = make_float2(-INFINITY, 0.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TcCfg<BN>::TMEM_COLS));
  }
}

// Merge the key splits of every (unit, row): O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One CTA per (unit, 8 dims), one thread per M row: the partials are stored
// row-innermost, so every load is a coalesced run over the rows; each thread
// requests all splits' data before combining.
constexpr int TC_MAX_SPLITS = 16;
constexpr int TC_LPT_MAX_REQ = 128;   // longest-first request order up to this batch (each CTA ranks them all)

template <int S, int D = TC_D>   // capacity for the number of splits (>= p.splits); head dim
__global__ void __launch_bounds__(128)
tree_attn_combine_kernel(const TcParams p) {
  const AttnGeom& g = p.g;
  const int groups = D / 8;
  int u = blockIdx.x / groups;
  const int rg = blockIdx.x - u * groups;
  const int unit = u;
  const int mt = u % p.mtiles; u /= p.mtiles;
  const int kvh = u % g.Hkv; u /= g.Hkv;
  const int r = u % g.n_req; u /= g.n_req;
  const int layer = u;
  const int nn = p.n_nodes[r];
  const int node0 = mt * (TC_BM / p.G);
  if (node0 >= nn) return;
  const int P = p.prefix_len[r];
  const long long cap = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
  if (P < 0 || (long long)P + nn > cap) return;
  const int row = threadIdx.x;                   // one M row per thread, 8 dims per CTA
  const int d0 = rg * 8;
  const int node = node0 + row / p.G;
  if (node >= nn) return;
  const int hq = kvh * p.G + row % p.G;
  // every split's statistics and partial row are requested before any is used
  float2 ml[S];
  float4 pa[S], pb[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s < p.splits) {
      const size_t slot = (size_t)unit * p.splits + s;
      ml[s] = p.ws_ml[slot * TC_BM + row];
      // partial O layout: [slot][D/4][128 rows] float4, so consecutive rows are consecutive
      const float4* wo = reinterpret_cast<const float4*>(p.ws_o) + (slot * (D / 4) + d0 / 4) * TC_BM + row;
      pa[s] = wo[0];
      pb[s] = wo[TC_BM];
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < S; ++s)
    if (s < p.splits) M = fmaxf(M, ml[s].x);
  float wsum = 0.f;
  float acc[8];
#pragma unroll
  for (int d = 0; d < 8; ++d) acc[d] = 0.f;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s < p.splits && ml[s].x != -INFINITY) {
      const float w = exp2f(ml[s].x - M);
      wsum += w * ml[s].y;
      acc[0] += w * pa[s].x; acc[1] += w * pa[s].y; acc[2] += w * pa[s].z; acc[3] += w * pa[s].w;
      acc[4] += w * pb[s].x; acc[5] += w * pb[s].y; acc[6] += w * pb[s].z; acc[7] += w * pb[s].w;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* orow = p.out + ((((size_t)layer * g.n_req + r) * g.n + node) * g.Hq + hq) * D + d0;
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(orow) = pk;
  if (p.out_lse && d0 == 0)
    p.out_lse[(((size_t)layer * g.n_req + r) * g.n + node) * g.Hq + hq] = (M + log2f(wsum)) * 0.6931471805599453f;
}

// ---------------------------------------------------------------- host side
struct TcPlan {
  int G, mtiles, splits, units, bn;
};

inline TcPlan tc_plan(const AttnGeom& g, int num_sms) {
  TcPlan pl;
  pl.G = g.Hq / g.Hkv;
  pl.mtiles = (g.n * pl.G + TC_BM - 1) / TC_BM;
  pl.units = g.layers * g.n_req * g.Hkv * pl.mtiles;
  // Split the key range only when the units alone leave CTA slots idle; a
  // split keeps at least TC_MIN_SPLIT_TILES key tiles to amortise its
  // set-up.  64-key tiles (two CTAs per SM) unless the split 128-key plan
  // leaves each CTA fewer than TC_SHORT_TILES tiles (short prefixes).
  const long long cap = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
  auto plan_splits = [&](int bn, int ctas, int min_tiles) {
    const int slots = num_sms * ctas;
    const long long tiles_cap = (cap + bn - 1) / bn;
    int splits = 1;
    if (pl.units < slots) {
      splits = slots / pl.units;
      if (splits > TC_MAX_SPLITS) splits = TC_MAX_SPLITS;
      if ((long long)splits * min_tiles > tiles_cap) splits = (int)(tiles_cap / min_tiles);
      if (splits < 1) splits = 1;
    }
    return splits;
  };
  const int s128 = plan_splits(128, TcCfg<128>::CTAS, 1);
  const long long t128 = (cap + 127) / 128;
  if (pl.units < num_sms && t128 / s128 < TC_SHORT_TILES) {
    pl.bn = 128;
    pl.splits = s128;
  } else {
    pl.bn = 64;
    pl.splits = plan_splits(64, TcCfg<64>::CTAS, TC_MIN_SPLIT_TILES);
  }
  return pl;
}

inline size_t tc_attn_ws_bytes(const AttnGeom& g, int num_sms) {
  TcPlan pl = tc_plan(g, num_sms);
  if (pl.splits == 1) return 0;
  const size_t slots = (size_t)pl.units * pl.splits;
  return align256(slots * TC_BM * TC_D * 4) + align256(slots * TC_BM * 8);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// 4-D bf16 map over (D, dim1, dim2, dim3) with a (64, b1, b2, 1) box and 128B swizzle.
inline bool make_map_4d(CUtensorMap* m, const void* base, uint64_t d1, uint64_t d2, uint64_t d3, uint32_t b1,
                        uint32_t b2, uint64_t D = TC_D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {D, d1, d2, d3};
  cuuint64_t strides[3] = {D * 2, D * 2 * d1, D * 2 * d1 * d2};
  cuuint32_t box[4] = {64, b1, b2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

inline int tc_attn_launch(const void* q, const void* kc, const void* vc, const int32_t* block_table,
                          const int32_t* prefix_len, const uint32_t* anc, const int32_t* n_nodes, const AttnGeom& g,
                          void* out, float* out_lse, void* ws, int num_sms, cudaStream_t stream,
                          uint64_t wait_ns = 0, int stop_tile = -1, int early = 0) {
  TcPlan pl = tc_plan(g, num_sms);
  TcParams p;
  p.g = g;
  p.G = pl.G;
  p.mtiles = pl.mtiles;
  p.splits = pl.splits;
  p.units = pl.units;
  p.block_table = block_table;
  p.prefix_len = prefix_len;
  p.anc = anc;
  p.n_nodes = n_nodes;
  p.out = (__nv_bfloat16*)out;
  p.out_lse = out_lse;
  p.ws_o = nullptr;
  p.ws_ml = nullptr;
  p.lpt = (pl.splits == 1 && g.n_req > 1 && g.n_req <= TC_LPT_MAX_REQ) ? 1 : 0;
  p.wait_ns = wait_ns > 0 ? wait_ns : TC_WAIT_NS;
  p.stop_tile = stop_tile;
  p.early = (early && !g.paged && !p.lpt) ? 1 : 0;   // start during the build (see the kernel)
  if (pl.splits > 1) {
    const size_t slots = (size_t)pl.units * pl.splits;
    p.ws_o = (float*)ws;
    p.ws_ml = (float2*)((char*)ws + align256(slots * TC_BM * TC_D * 4));
  }
  CUtensorMap mq, mk, mv;
  if (!make_map_4d(&mq, q, (uint64_t)g.Hq, (uint64_t)g.n, (uint64_t)g.layers * g.n_req, (uint32_t)pl.G,
                   (uint32_t)(TC_BM / pl.G)))
    return DDTREE_ERR_CUDA;
  if (!g.paged) {
    if (!make_map_4d(&mk, kc, g.Hkv, g.s_max, (uint64_t)g.layers * g.n_req, 1, pl.bn)) return DDTREE_ERR_CUDA;
    if (!make_map_4d(&mv, vc, g.Hkv, g.s_max, (uint64_t)g.layers * g.n_req, 1, pl.bn)) return DDTREE_ERR_CUDA;
  } else {
    if (!make_map_4d(&mk, kc, g.Hkv, DDTREE_PAGE, (uint64_t)g.layers * g.num_blocks, 1, DDTREE_PAGE))
      return DDTREE_ERR_CUDA;
    if (!make_map_4d(&mv, vc, g.Hkv, DDTREE_PAGE, (uint64_t)g.layers * g.num_blocks, 1, DDTREE_PAGE))
      return DDTREE_ERR_CUDA;
  }
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(tree_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc_smem_bytes<128>()) != cudaSuccess ||
        cudaFuncSetAttribute(tree_attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tc_smem_bytes<64>()) != cudaSuccess)
      return DDTREE_ERR_CUDA;
    attr_set = true;
  }
  const long long grid = (long long)pl.units * pl.splits;
  if (grid > 0x7fffffffLL) return DDTREE_ERR_UNSUPPORTED;
  const cudaError_t le =
      pl.bn == 64 ? launch_maybe_pdl(tree_attn_tc_kernel<64>, dim3((unsigned)grid), dim3(TC_THREADS),
                                     tc_smem_bytes<64>(), stream, p.early != 0, mq, mk, mv, p)
                  : launch_maybe_pdl(tree_attn_tc_kernel<128>, dim3((unsigned)grid), dim3(TC_THREADS),
                                     tc_smem_bytes<128>(), stream, p.early != 0, mq, mk, mv, p);
  if (le != cudaSuccess || cudaGetLastError() != cudaSuccess) return DDTREE_ERR_CUDA;
  if (pl.splits > 1) {
    if (pl.splits <= 8)
      tree_attn_combine_kernel<8><<<pl.units * (TC_D / 8), TC_BM, 0, stream>>>(p);
    else
      tree_attn_combine_kernel<TC_MAX_SPLITS><<<pl.units * (TC_D / 8), TC_BM, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return DDTREE_ERR_CUDA;
  }
  return DDTREE_OK;
}

}  // namespace ddt
