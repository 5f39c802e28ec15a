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
// lexicographically ascending.  The heap of Proposition 3 pops the
// prefixes in exactly that order.
//
// Design: one CTA per request; one warp runs the queue, the whole CTA
// writes the outputs.  Instead of one pop per step the warp pops in rounds:
//  * the frontier (the heap's contents) is kept sorted in shared memory;
//  * a round takes its m = min(32, frontier, remaining budget) best entries;
//    call the m-th one tau.  Every prefix that will ever be popped before
//    tau is one of those entries or is generated from them by sibling/child
//    pushes (a generated entry never beats its generator), so the round
//    expands that closure level by level, keeping generated entries that
//    beat tau and setting the others aside;
//  * the closure is sorted (bitonic, one warp) and popped as consecutive
//    nodes; the set-aside entries are sorted and merged into the frontier.
// The pop sequence is exactly the heap's; a round replaces up to dozens of
// dependent heap steps.  If a closure outgrows its buffer the round is
// redone with a smaller m (m = 1 always fits: nothing beats its generator).
//
// Order keys are 64 bits: the fp32 score's order key, then a tie key that
// packs the tuple's first ranks (exactly equal fp32 scores are common with
// bf16 logits: 45-65% of popped prefixes share a score).  Only entries that
// agree on score and on every packed rank fall back to an exact rank-tuple
// comparison that walks parent pointers to the common ancestor.
#pragma once

#include "common.cuh"

namespace ddt {

constexpr int BUILD_THREADS = 256;
constexpr int BUILD_MAXM = 32;          // frontier entries taken per round
constexpr int BUILD_CCAP = 128;         // closure capacity per round
constexpr int BUILD_NCAP = 2 * BUILD_CCAP;

// Entry metadata: parent node (11 bits), depth (6 bits), rank (15 bits).
__device__ __forceinline__ uint32_t pack_meta(int parent, int depth, int rank) {
  return (uint32_t)parent | ((uint32_t)depth << 11) | ((uint32_t)rank << 17);
}
__device__ __forceinline__ int meta_parent(uint32_t m) { return (int)(m & 0x7FFu); }
__device__ __forceinline__ int meta_depth(uint32_t m) { return (int)((m >> 11) & 0x3Fu); }
__device__ __forceinline__ int meta_rank(uint32_t m) { return (int)(m >> 17); }

__device__ __forceinline__ uint32_t score_key(float s) { return key32_of_f32(s); }

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

inline TieCode tie_code(int kc, int L) {
  TieCode t;
  t.tbits = 1;
  while ((1 << t.tbits) <= kc) ++t.tbits;      // fields hold rank + 1 <= kc
  t.tdepth = 32 / t.tbits;
  if (t.tdepth > L) t.tdepth = L;
  return t;
}

// Exact lexicographic comparison of two entries' rank tuples (a proper
// prefix is smaller).  Walks the parent chains: lift the deeper entry to the
// other's depth, then both to their common parent, and compare the ranks
// just below it.
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

// The entry arrays of one list (frontier, closure or set-aside entries).
struct EntryList {
  uint32_t* kx;    // score key
  uint32_t* ky;    // tie key
  float* sc;       // score
  float* ps;       // score of the parent node
  uint32_t* mt;    // packed parent/depth/rank
};

struct BuildCtx {
  const int* nd_parent;
  const int* nd_rank;
  // a before b in the pop order
  __device__ __forceinline__ bool before(uint32_t ax, uint32_t ay, uint32_t am, uint32_t bx, uint32_t by,
                                         uint32_t bm) const {
    if (ax != bx) return ax > bx;
    if (ay != by) return ay > by;
    return tuple_less(am, bm, nd_parent, nd_rank);
  }
};

// Warp bitonic sort of indices idx[0..len) into pop order (best first);
// padding up to a power of two with -1, which sorts last.
__device__ __forceinline__ int warp_sort(int* idx, int len, const EntryList& e, const BuildCtx& cx, int lane) {
  int p2 = 1;
  while (p2 < len) p2 <<= 1;
  for (int i = len + lane; i < p2; i += 32) idx[i] = -1;
  __syncwarp();
  for (int size = 2; size <= p2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < p2 / 2; i += 32) {
        const int lo = 2 * stride * (i / stride) + (i % stride);
        const int hi = lo + stride;
        const int a = idx[lo], b = idx[hi];
        // desc: best first within blocks whose (lo & size) == 0
        bool b_first;
        if (a < 0) b_first = b >= 0;
        else if (b < 0) b_first = false;
        else b_first = cx.before(e.kx[b], e.ky[b], e.mt[b], e.kx[a], e.ky[a], e.mt[a]);
        const bool asc = (lo & size) != 0;
        if (b_first != asc) { idx[lo] = b; idx[hi] = a; }
      }
      __syncwarp();
    }
  }
  return p2;
}

struct BuildSmem {
  float* lp;                 // [L][kc]
  EntryList F0, F1;          // frontier, double buffered, sorted best first [n + 1]
  EntryList C;               // closure of the current round [CCAP]
  EntryList N;               // entries set aside this round [NCAP]
  int* cidx;                 // [CCAP] sort permutation of C
  int* cinv;                 // [CCAP] sorted position of each closure entry
  int* nidx;                 // [NCAP] sort permutation of N
  int* nins;                 // [NCAP] insertion point of each sorted N entry in the frontier
  int* nd_parent;            // [n + CCAP] (provisional ids during a round)
  int* nd_rank;
  int* nd_depth;
  float* nd_score;
};

inline size_t build_smem_bytes(int L, int kc, int B) {
  const size_t n = (size_t)B + 1;
  const size_t entry = 5 * 4;
  return (size_t)L * kc * 4 + 2 * (n + 1) * entry + (BUILD_CCAP + BUILD_NCAP) * entry +
         (2 * BUILD_CCAP + 2 * BUILD_NCAP) * 4 + (n + BUILD_CCAP) * 4 * 4;
}

__device__ __forceinline__ EntryList carve_list(unsigned char*& p, int cap) {
  EntryList e;
  e.kx = (uint32_t*)p; p += (size_t)cap * 4;
  e.ky = (uint32_t*)p; p += (size_t)cap * 4;
  e.sc = (float*)p;    p += (size_t)cap * 4;
  e.ps = (float*)p;    p += (size_t)cap * 4;
  e.mt = (uint32_t*)p; p += (size_t)cap * 4;
  return e;
}

__device__ __forceinline__ void put(const EntryList& e, int i, uint32_t kx, uint32_t ky, float sc, float ps,
                                    uint32_t mt) {
  e.kx[i] = kx; e.ky[i] = ky; e.sc[i] = sc; e.ps[i] = ps; e.mt[i] = mt;
}
__device__ __forceinline__ void copy_entry(const EntryList& d, int i, const EntryList& s, int j) {
  d.kx[i] = s.kx[j]; d.ky[i] = s.ky[j]; d.sc[i] = s.sc[j]; d.ps[i] = s.ps[j]; d.mt[i] = s.mt[j];
}

__global__ void __launch_bounds__(BUILD_THREADS, 1)
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
    sm.lp = (float*)p; p += (size_t)L * kc * 4;
    sm.F0 = carve_list(p, n + 1);
    sm.F1 = carve_list(p, n + 1);
    sm.C = carve_list(p, BUILD_CCAP);
    sm.N = carve_list(p, BUILD_NCAP);
    sm.cidx = (int*)p; p += BUILD_CCAP * 4;
    sm.cinv = (int*)p; p += BUILD_CCAP * 4;
    sm.nidx = (int*)p; p += BUILD_NCAP * 4;
    sm.nins = (int*)p; p += BUILD_NCAP * 4;
    sm.nd_parent = (int*)p; p += (size_t)(n + BUILD_CCAP) * 4;
    sm.nd_rank = (int*)p;   p += (size_t)(n + BUILD_CCAP) * 4;
    sm.nd_depth = (int*)p;  p += (size_t)(n + BUILD_CCAP) * 4;
    sm.nd_score = (float*)p;
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
    const BuildCtx cx{sm.nd_parent, sm.nd_rank};
    if (lane == 0) {
      sm.nd_parent[0] = -1;
      sm.nd_rank[0] = -1;
      sm.nd_depth[0] = 0;
      sm.nd_score[0] = 0.f;
    }
    int cur = 0, nf = 0, pops = 0;
    if (B > 0) {   // the frontier starts with the best token of position 1
      if (lane == 0) {
        const float s0 = __fadd_rn(0.f, sm.lp[0]);
        put(sm.F0, 0, score_key(s0), ~tc.unit(1), s0, 0.f, pack_meta(0, 1, 0));
      }
      nf = 1;
    }
    __syncwarp();
    int mcap = BUILD_MAXM;
    while (pops < B && nf > 0) {
      const EntryList F = cur ? sm.F1 : sm.F0;
      int m = min(min(mcap, nf), B - pops);
      const uint32_t tx = F.kx[m - 1], ty = F.ky[m - 1], tm = F.mt[m - 1];   // tau
      const int base = pops + 1;            // provisional id of closure entry c is base + c
      // ---- closure: the m best entries, then everything they generate that beats tau ----
      for (int c = lane; c < m; c += 32) {
        copy_entry(sm.C, c, F, c);
        const uint32_t mt = F.mt[c];
        sm.nd_parent[base + c] = meta_parent(mt);
        sm.nd_rank[base + c] = meta_rank(mt);
        sm.nd_depth[base + c] = meta_depth(mt);
      }
      __syncwarp();
      int nc = m, nn = 0, lo = 0;
      bool overflow = false;
      while (lo < nc && !overflow) {
        const int hi = nc;
        for (int c0 = lo; c0 < hi; c0 += 32) {
          const int c = c0 + lane;
          uint32_t gx[2] = {0u, 0u}, gy[2], gm[2];
          float gs[2], gp[2];
          bool gv[2] = {false, false};
          if (c < hi) {
            const uint32_t mt = sm.C.mt[c];
            const int d = meta_depth(mt), rk = meta_rank(mt), par = meta_parent(mt);
            const uint32_t packed = ~sm.C.ky[c];
            const float s = sm.C.sc[c], ps = sm.C.ps[c];
            if (rk + 1 < kc) {         // next sibling
              gs[0] = __fadd_rn(ps, sm.lp[(d - 1) * kc + rk + 1]);
              gx[0] = score_key(gs[0]); gy[0] = ~(packed + tc.unit(d)); gp[0] = ps;
              gm[0] = pack_meta(par, d, rk + 1); gv[0] = true;
            }
            if (d < L) {               // first child
              gs[1] = __fadd_rn(s, sm.lp[d * kc]);
              gx[1] = score_key(gs[1]); gy[1] = ~(packed + tc.unit(d + 1)); gp[1] = s;
              gm[1] = pack_meta(base + c, d + 1, 0); gv[1] = true;
            }
          }
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const bool to_c = gv[g] && cx.before(gx[g], gy[g], gm[g], tx, ty, tm);
            const bool to_n = gv[g] && !to_c;
            const unsigned bc = __ballot_sync(0xffffffffu, to_c);
            const unsigned bn = __ballot_sync(0xffffffffu, to_n);
            const unsigned below = (1u << lane) - 1u;
            if (nc + __popc(bc) > BUILD_CCAP || nn + __popc(bn) > BUILD_NCAP) {
              overflow = true;
            } else {
              if (to_c) {
                const int ci = nc + __popc(bc & below);
                put(sm.C, ci, gx[g], gy[g], gs[g], gp[g], gm[g]);
                sm.nd_parent[base + ci] = meta_parent(gm[g]);
                sm.nd_rank[base + ci] = meta_rank(gm[g]);
                sm.nd_depth[base + ci] = meta_depth(gm[g]);
              }
              if (to_n) put(sm.N, nn + __popc(bn & below), gx[g], gy[g], gs[g], gp[g], gm[g]);
              nc += __popc(bc);
              nn += __popc(bn);
            }
          }
          __syncwarp();
          if (overflow) break;
        }
        lo = hi;
      }
      if (overflow) {             // redo the round with fewer entries
        mcap = max(1, m / 2);
        __syncwarp();
        continue;
      }
      mcap = BUILD_MAXM;
      // ---- pop the closure in order ----
      for (int c = lane; c < nc; c += 32) sm.cidx[c] = c;
      __syncwarp();
      warp_sort(sm.cidx, nc, sm.C, cx, lane);
      for (int s = lane; s < nc; s += 32) sm.cinv[sm.cidx[s]] = s;
      __syncwarp();
      const int npop = min(nc, B - pops);
      int pv[4], rv[4], dv[4];
      float sv[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {     // read every provisional record before writing final ones
        const int s = lane + 32 * t;
        if (s < npop) {
          const int c = sm.cidx[s];
          const uint32_t mt = sm.C.mt[c];
          int p = meta_parent(mt);
          if (p >= base) p = base + sm.cinv[p - base];
          pv[t] = p; rv[t] = meta_rank(mt); dv[t] = meta_depth(mt); sv[t] = sm.C.sc[c];
        }
      }
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int s = lane + 32 * t;
        if (s < npop) {
          sm.nd_parent[base + s] = pv[t];
          sm.nd_rank[base + s] = rv[t];
          sm.nd_depth[base + s] = dv[t];
          sm.nd_score[base + s] = sv[t];
        }
      }
      pops += npop;
      __syncwarp();
      if (pops >= B) break;
      // ---- set-aside entries: final parent ids, sort, merge into the rest of the frontier ----
      for (int j = lane; j < nn; j += 32) {
        const uint32_t mt = sm.N.mt[j];
        const int p = meta_parent(mt);
        if (p >= base) sm.N.mt[j] = pack_meta(base + sm.cinv[p - base], meta_depth(mt), meta_rank(mt));
        sm.nidx[j] = j;
      }
      __syncwarp();
      warp_sort(sm.nidx, nn, sm.N, cx, lane);
      const int nrest = nf - m;
      // insertion point of each sorted set-aside entry among the remaining frontier F[m..nf)
      for (int j = lane; j < nn; j += 32) {
        const int e = sm.nidx[j];
        int a = 0, b = nrest;
        while (a < b) {
          const int mid = (a + b) >> 1;
          const int fi = m + mid;
          if (cx.before(F.kx[fi], F.ky[fi], F.mt[fi], sm.N.kx[e], sm.N.ky[e], sm.N.mt[e])) a = mid + 1;
          else b = mid;
        }
        sm.nins[j] = a;
      }
      __syncwarp();
      const EntryList G = cur ? sm.F0 : sm.F1;
      for (int j = lane; j < nn; j += 32) copy_entry(G, sm.nins[j] + j, sm.N, sm.nidx[j]);
      for (int i = lane; i < nrest; i += 32) {
        int a = 0, b = nn;              // set-aside entries placed before frontier entry i
        while (a < b) {
          const int mid = (a + b) >> 1;
          if (sm.nins[mid] <= i) a = mid + 1;
          else b = mid;
        }
        copy_entry(G, i + a, F, m + i);
      }
      nf = nrest + nn;
      cur ^= 1;
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

}  // namespace ddt
