// Stage 2: best-first tree build over rank tuples.
//
// "DDTree Deep Dive" §2: Proposition 3 (a max-heap over rank tuples that
// pops the best prefix and pushes its next sibling and its first child
// yields exactly the top-B prefixes), Proposition 2 (they form a
// prefix-closed optimal tree); §3 (tree_indices = [position, parent]);
// §4 (ancestor-only visibility, rebuilt every round).
//
// Order of prefixes: fp32 score (sum of lp in root-to-leaf order, one
// correctly rounded add per depth) descending, then rank tuple
// lexicographically ascending.  Under that order every pop is the
// frontier's maximum, so the kernel only needs a priority queue with an
// exact total order.
//
// Design: one CTA per request.  The lp table (ranks < min(K, B)) is staged
// in shared memory.  Warp 0 runs the queue: frontier slot s lives in
// shared memory and belongs to lane s % 32, and every lane caches its best
// entry (order key, score, parent score, packed parent/depth/rank) in
// registers.  The order key of an entry is 64 bits: the fp32 score's order
// key, then a tie key that packs the tuple's first ranks (exactly equal fp32
// scores are common with bf16 logits: 45-65% of popped prefixes share a
// score).  A pop is two `redux.sync.max` rounds and a ballot plus four
// shuffles, with no shared-memory read of the popped entry; only entries
// that agree on score and on every packed rank fall back to an exact
// rank-tuple comparison that walks parent pointers to the common ancestor.  A popped slot is reused for the popped
// entry's next sibling, so only the popped entry's lane rescans its slots
// and the child's lane compares one entry.  After the pops every thread
// writes one node row and builds its ancestor bitmask by walking its
// parent chain (at most L+1 nodes).
#pragma once

#include "common.cuh"

namespace ddt {

constexpr int BUILD_THREADS = 512;

// Frontier entry metadata: parent node (11 bits), depth (6 bits), rank (11 bits).
__device__ __forceinline__ uint32_t pack_meta(int parent, int depth, int rank) {
  return (uint32_t)parent | ((uint32_t)depth << 11) | ((uint32_t)rank << 17);
}
__device__ __forceinline__ int meta_parent(uint32_t m) { return (int)(m & 0x7FFu); }
__device__ __forceinline__ int meta_depth(uint32_t m) { return (int)((m >> 11) & 0x3Fu); }
__device__ __forceinline__ int meta_rank(uint32_t m) { return (int)(m >> 17); }

// Score order key; 0 marks an empty slot (every real score, -inf included,
// has a larger key).
__device__ __forceinline__ uint32_t score_key(float s) { return key32_of_f32(s); }

struct BuildSmem {
  float* lp;          // [L][kc]
  uint2* fr_key;      // [B+1] (score key, tie key); (0,0) = empty slot
  float* fr_score;    // [B+1]
  float* fr_pscore;   // [B+1] score of the entry's parent node
  uint32_t* fr_meta;  // [B+1]
  int* nd_parent;     // [B+1]
  int* nd_rank;       // [B+1]
  int* nd_depth;      // [B+1]
  float* nd_score;    // [B+1]
};

// Tie key: the first `tdepth` ranks of the tuple packed as (rank + 1) in
// `tbits`-bit fields, most significant first, absent depths 0, then
// complemented.  Between entries with equal scores, a larger tie key means a
// lexicographically smaller tuple (a proper prefix is smaller than its
// extensions); equal tie keys mean the first tdepth ranks agree.
struct TieCode {
  int tbits, tdepth;
  __device__ __forceinline__ uint32_t unit(int depth) const {   // +1 at the field of this depth (1-based)
    return depth <= tdepth ? (1u << (tbits * (tdepth - depth))) : 0u;
  }
};

// Exact lexicographic comparison of two frontier entries' rank tuples (a
// proper prefix is smaller), for the rare case of equal scores and equal tie
// keys.  Walks the parent chains: lift the deeper entry to the other's depth,
// then both to their common parent, and compare the ranks just below it.
__device__ __forceinline__ bool tuple_less(uint32_t ma, uint32_t mb, const int* nd_parent, const int* nd_rank) {
  int pa = meta_parent(ma), ra = meta_rank(ma), da = meta_depth(ma);
  int pb = meta_parent(mb), rb = meta_rank(mb), db = meta_depth(mb);
  const bool a_shorter = da < db;
  while (da > db) { ra = nd_rank[pa]; pa = nd_parent[pa]; --da; }
  while (db > da) { rb = nd_rank[pb]; pb = nd_parent[pb]; --db; }
  if (pa == pb && ra == rb) return a_shorter;   // one tuple is a prefix of the other
  while (pa != pb) {
    ra = nd_rank[pa]; pa = nd_parent[pa];
    rb = nd_rank[pb]; pb = nd_parent[pb];
  }
  return ra < rb;
}

// a before b in the pop order: larger score key, then larger tie key, then
// (both equal) the smaller rank tuple.
__device__ __forceinline__ bool entry_before(uint2 ka, uint32_t ma, uint2 kb, uint32_t mb, const int* nd_parent,
                                             const int* nd_rank) {
  if (ka.x != kb.x) return ka.x > kb.x;
  if (ka.y != kb.y) return ka.y > kb.y;
  return tuple_less(ma, mb, nd_parent, nd_rank);
}

__global__ void __launch_bounds__(BUILD_THREADS)
build_kernel(const int32_t* __restrict__ ids, const float* __restrict__ lp,
             const int32_t* __restrict__ root_token, int L, int K, int B, int kc, TieCode tc,
             int32_t* __restrict__ node_token, int32_t* __restrict__ parent,
             int32_t* __restrict__ depth, int32_t* __restrict__ node_rank,
             float* __restrict__ score, uint32_t* __restrict__ anc, int32_t* __restrict__ n_nodes) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  const int n = B + 1;
  const int W = (n + 31) >> 5;

  BuildSmem sm;
  {
    unsigned char* p = smem_raw;
    sm.fr_key = (uint2*)p;      p += (size_t)n * 8;
    sm.lp = (float*)p;          p += (size_t)L * kc * 4;
    sm.fr_score = (float*)p;    p += (size_t)n * 4;
    sm.fr_pscore = (float*)p;   p += (size_t)n * 4;
    sm.fr_meta = (uint32_t*)p;  p += (size_t)n * 4;
    sm.nd_parent = (int*)p;     p += (size_t)n * 4;
    sm.nd_rank = (int*)p;       p += (size_t)n * 4;
    sm.nd_depth = (int*)p;      p += (size_t)n * 4;
    sm.nd_score = (float*)p;    p += (size_t)n * 4;
  }
  __shared__ int s_pops;

  // stage the lp table (only ranks < kc can ever be popped)
  const float* lpr = lp + (size_t)r * L * K;
  for (int i = tid; i < L * kc; i += BUILD_THREADS) {
    const int d = i / kc, k = i - d * kc;
    sm.lp[i] = lpr[(size_t)d * K + k];
  }
  __syncthreads();

  if (tid < 32) {
    const int lane = tid;
    if (lane == 0) {
      sm.nd_parent[0] = -1;
      sm.nd_rank[0] = -1;
      sm.nd_depth[0] = 0;
      sm.nd_score[0] = 0.f;
    }
    // this lane's best frontier entry, cached in registers (bkey (0,0): none)
    uint2 bkey = make_uint2(0u, 0u);
    uint32_t bmeta = 0;
    float bscore = 0.f, bpscore = 0.f;
    int bslot = -1;
    int next_slot = 0;
    if (B > 0) {   // the frontier starts with the best token of position 1
      const float s0 = __fadd_rn(0.f, sm.lp[0]);
      if (lane == 0) {
        bkey = make_uint2(score_key(s0), ~tc.unit(1));
        bmeta = pack_meta(0, 1, 0);
        bscore = s0;
        bpscore = 0.f;
        bslot = 0;
        sm.fr_key[0] = bkey;
        sm.fr_score[0] = s0;
        sm.fr_pscore[0] = 0.f;
        sm.fr_meta[0] = bmeta;
      }
      next_slot = 1;
    }
    __syncwarp();
    int pops = 0;
    while (pops < B) {
      // the frontier's best entry: max score key, then max tie key, then (rare) tuple walk
      const uint32_t mhi = __reduce_max_sync(0xffffffffu, bkey.x);
      if (mhi == 0) break;   // frontier empty
      const uint32_t mlo = __reduce_max_sync(0xffffffffu, bkey.x == mhi ? bkey.y : 0u);
      unsigned ties = __ballot_sync(0xffffffffu, bkey.x == mhi && bkey.y == mlo);
      int wl = __ffs(ties) - 1;
      ties &= ties - 1;
      if (ties) {
        uint32_t wm = __shfl_sync(0xffffffffu, bmeta, wl);
        while (ties) {
          const int l2 = __ffs(ties) - 1;
          ties &= ties - 1;
          const uint32_t m2 = __shfl_sync(0xffffffffu, bmeta, l2);
          if (tuple_less(m2, wm, sm.nd_parent, sm.nd_rank)) { wl = l2; wm = m2; }
        }
      }
      const uint32_t meta = __shfl_sync(0xffffffffu, bmeta, wl);
      const float sc = __shfl_sync(0xffffffffu, bscore, wl);
      const float ps = __shfl_sync(0xffffffffu, bpscore, wl);
      const int slot = __shfl_sync(0xffffffffu, bslot, wl);
      const uint32_t packed = ~mlo;                         // the popped entry's packed ranks
      const int par = meta_parent(meta), d = meta_depth(meta), rk = meta_rank(meta);
      const int node = ++pops;
      const bool sib = rk + 1 < kc;              // next sibling: same parent, next rank
      const bool child = d < L;                  // first child: one position deeper
      const float lsib = sib ? sm.lp[(d - 1) * kc + rk + 1] : 0.f;
      const float lchild = child ? sm.lp[d * kc] : 0.f;
      if (lane == 0) {
        sm.nd_parent[node] = par;
        sm.nd_rank[node] = rk;
        sm.nd_depth[node] = d;
        sm.nd_score[node] = sc;
      }
      const float ssib = __fadd_rn(ps, lsib);
      const float schild = __fadd_rn(sc, lchild);
      const uint2 ksib = sib ? make_uint2(score_key(ssib), ~(packed + tc.unit(d))) : make_uint2(0u, 0u);
      const uint2 kchild = make_uint2(score_key(schild), ~(packed + tc.unit(d + 1)));
      const uint32_t msib = pack_meta(par, d, rk + 1), mchild = pack_meta(node, d + 1, 0);
      const int cslot = next_slot;
      if (child) ++next_slot;
      const int sl = slot & 31, cl = cslot & 31;
      if (lane == sl) {
        sm.fr_key[slot] = ksib;
        sm.fr_score[slot] = ssib;
        sm.fr_pscore[slot] = ps;
        sm.fr_meta[slot] = msib;
      }
      if (child && lane == cl) {
        sm.fr_key[cslot] = kchild;
        sm.fr_score[cslot] = schild;
        sm.fr_pscore[cslot] = sc;
        sm.fr_meta[cslot] = mchild;
      }
      __syncwarp();
      if (lane == sl) {          // this lane's best was popped: rescan its slots
        bkey = make_uint2(0u, 0u);
        bslot = -1;
        for (int s2 = lane; s2 < next_slot; s2 += 32) {
          const uint2 k = sm.fr_key[s2];
          if (k.x == 0) continue;
          if (bslot < 0 || entry_before(k, sm.fr_meta[s2], bkey, bmeta, sm.nd_parent, sm.nd_rank)) {
            bkey = k;
            bslot = s2;
            bmeta = sm.fr_meta[s2];
          }
        }
        if (bslot >= 0) {
          bscore = sm.fr_score[bslot];
          bpscore = sm.fr_pscore[bslot];
        }
      } else if (child && lane == cl) {
        if (bslot < 0 || entry_before(kchild, mchild, bkey, bmeta, sm.nd_parent, sm.nd_rank)) {
          bkey = kchild;
          bslot = cslot;
          bmeta = mchild;
          bscore = schild;
          bpscore = sc;
        }
      }
    }
    if (lane == 0) s_pops = pops;
  }
  __syncthreads();

  // ---- outputs ----
  const int nn = s_pops + 1;
  const size_t ro = (size_t)r * n;
  const int32_t* idr = ids + (size_t)r * L * K;
  for (int i = tid; i < n; i += BUILD_THREADS) {
    const bool live = i < nn;
    const int d = live ? sm.nd_depth[i] : -1;
    const int rk = live ? sm.nd_rank[i] : -1;
    if (node_token) node_token[ro + i] = !live ? -1 : (i == 0 ? root_token[r] : idr[(size_t)(d - 1) * K + rk]);
    parent[ro + i] = live ? sm.nd_parent[i] : -1;
    if (depth) depth[ro + i] = d;
    if (node_rank) node_rank[ro + i] = rk;
    if (score) score[ro + i] = live ? sm.nd_score[i] : -INFINITY;
    // ancestor-or-self bitmask: walk up the chain, words from high to low
    uint32_t* arow = anc + ro * W + (size_t)i * W;
    int j = live ? i : -1;
    for (int w = W - 1; w >= 0; --w) {
      uint32_t acc = 0;
      while (j >= 0 && (j >> 5) == w) {
        acc |= 1u << (j & 31);
        j = sm.nd_parent[j];
      }
      arow[w] = acc;
    }
  }
  if (tid == 0) n_nodes[r] = nn;
}

inline TieCode tie_code(int kc, int L) {
  TieCode t;
  t.tbits = 1;
  while ((1 << t.tbits) <= kc) ++t.tbits;      // fields hold rank + 1 <= kc
  t.tdepth = 32 / t.tbits;
  if (t.tdepth > L) t.tdepth = L;
  return t;
}

inline size_t build_smem_bytes(int L, int kc, int B) {
  return (size_t)L * kc * 4 + (size_t)(B + 1) * (8 + 4 * 7);
}

}  // namespace ddt
