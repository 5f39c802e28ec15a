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
// shared memory and belongs to lane s % 32, every lane caches the best of
// its slots, and a pop is one `redux.sync.max` over the lanes' 32-bit order
// keys plus a ballot.  Equal keys (equal fp32 scores) fall back to an exact
// rank-tuple comparison that walks parent pointers.  A popped slot is
// reused for the popped entry's next sibling, so only two lanes ever
// rescan.  After the pops every thread writes one node row and builds its
// ancestor bitmask by walking its parent chain (at most L+1 nodes).
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
  uint32_t* fr_key;   // [B+1]
  float* fr_score;    // [B+1]
  uint32_t* fr_meta;  // [B+1]
  int* nd_parent;     // [B+1]
  int* nd_rank;       // [B+1]
  int* nd_depth;      // [B+1]
  float* nd_score;    // [B+1]
};

// True iff the rank tuple of entry a is lexicographically smaller than b's
// (a proper prefix is smaller than its extensions).  Tuples are rebuilt
// from the parent chain; only used when two scores are exactly equal.
__device__ __noinline__ bool tuple_less(uint32_t ma, uint32_t mb, const int* nd_parent,
                                        const int* nd_rank) {
  int ta[33], tb[33];
  int da = meta_depth(ma), db = meta_depth(mb);
  ta[da - 1] = meta_rank(ma);
  for (int p = meta_parent(ma), k = da - 2; k >= 0; --k) { ta[k] = nd_rank[p]; p = nd_parent[p]; }
  tb[db - 1] = meta_rank(mb);
  for (int p = meta_parent(mb), k = db - 2; k >= 0; --k) { tb[k] = nd_rank[p]; p = nd_parent[p]; }
  int n = da < db ? da : db;
  for (int k = 0; k < n; ++k)
    if (ta[k] != tb[k]) return ta[k] < tb[k];
  return da < db;
}

__global__ void __launch_bounds__(BUILD_THREADS)
build_kernel(const int32_t* __restrict__ ids, const float* __restrict__ lp,
             const int32_t* __restrict__ root_token, int L, int K, int B, int kc,
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
    sm.lp = (float*)p;          p += (size_t)L * kc * 4;
    sm.fr_key = (uint32_t*)p;   p += (size_t)n * 4;
    sm.fr_score = (float*)p;    p += (size_t)n * 4;
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
    int d = i / kc, k = i - d * kc;
    sm.lp[i] = lpr[(size_t)d * K + k];
  }
  for (int i = tid; i < n; i += BUILD_THREADS) sm.fr_key[i] = 0;
  __syncthreads();

  if (tid < 32) {
    const int lane = tid;
    // root
    if (lane == 0) {
      sm.nd_parent[0] = -1;
      sm.nd_rank[0] = -1;
      sm.nd_depth[0] = 0;
      sm.nd_score[0] = 0.f;
    }
    int next_slot = 0;
    uint32_t bkey = 0;
    int bslot = -1;
    if (B > 0) {
      // the frontier starts with the best token of position 1
      const float s0 = __fadd_rn(0.f, sm.lp[0]);
      if (lane == 0) {
        sm.fr_key[0] = score_key(s0);
        sm.fr_score[0] = s0;
        sm.fr_meta[0] = pack_meta(0, 1, 0);
        bkey = score_key(s0);
        bslot = 0;
      }
      next_slot = 1;
    }
    __syncwarp();
    int pops = 0;
    while (pops < B) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, bkey);
      if (m == 0) break;   // frontier empty
      unsigned ties = __ballot_sync(0xffffffffu, bkey == m);
      int wl = __ffs(ties) - 1;
      int slot = __shfl_sync(0xffffffffu, bslot, wl);
      ties &= ties - 1;
      while (ties) {       // equal scores in several lanes: smallest rank tuple wins
        const int l2 = __ffs(ties) - 1;
        ties &= ties - 1;
        const int s2 = __shfl_sync(0xffffffffu, bslot, l2);
        if (tuple_less(sm.fr_meta[s2], sm.fr_meta[slot], sm.nd_parent, sm.nd_rank)) slot = s2;
      }
      const uint32_t meta = sm.fr_meta[slot];
      const float sc = sm.fr_score[slot];
      const int par = meta_parent(meta), d = meta_depth(meta), rk = meta_rank(meta);
      const int node = ++pops;
      if (lane == 0) {
        sm.nd_parent[node] = par;
        sm.nd_rank[node] = rk;
        sm.nd_depth[node] = d;
        sm.nd_score[node] = sc;
      }
      // next sibling replaces the popped entry in its slot
      const bool sib = rk + 1 < kc;
      const float ssib = sib ? __fadd_rn(sm.nd_score[par], sm.lp[(d - 1) * kc + rk + 1]) : 0.f;
      // first child goes to a fresh slot
      const bool child = d < L;
      const float schild = child ? __fadd_rn(sc, sm.lp[d * kc]) : 0.f;
      const int cslot = next_slot;
      if (child) ++next_slot;
      const int sl = slot & 31, cl = cslot & 31;
      if (lane == sl) {
        sm.fr_key[slot] = sib ? score_key(ssib) : 0u;
        sm.fr_score[slot] = ssib;
        sm.fr_meta[slot] = pack_meta(par, d, rk + 1);
      }
      if (child && lane == cl) {
        sm.fr_key[cslot] = score_key(schild);
        sm.fr_score[cslot] = schild;
        sm.fr_meta[cslot] = pack_meta(node, d + 1, 0);
      }
      __syncwarp();
      if (lane == sl) {          // rescan this lane's slots
        bkey = 0;
        bslot = -1;
        for (int s = lane; s < next_slot; s += 32) {
          const uint32_t k = sm.fr_key[s];
          if (k > bkey || (k != 0 && k == bkey &&
                           tuple_less(sm.fr_meta[s], sm.fr_meta[bslot], sm.nd_parent, sm.nd_rank))) {
            bkey = k;
            bslot = s;
          }
        }
      } else if (child && lane == cl) {
        const uint32_t k = sm.fr_key[cslot];
        if (k > bkey || (k == bkey && tuple_less(sm.fr_meta[cslot], sm.fr_meta[bslot], sm.nd_parent,
                                                 sm.nd_rank))) {
          bkey = k;
          bslot = cslot;
        }
      }
      __syncwarp();
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

inline size_t build_smem_bytes(int L, int kc, int B) {
  return (size_t)L * kc * 4 + (size_t)(B + 1) * 4 * 7;
}

}  // namespace ddt
