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
// writes the outputs.  The queue is a two-level tournament: frontier slot s
// (an entry of the heap) lives in shared memory in block s / 32, and the
// best entry of each block (its order key and slot) is cached in the
// registers of lane (block % 32).  A pop is a warp reduction over the cached
// block bests; the popped slot takes the popped entry's next sibling and the
// first child goes to a fresh slot, after which the one or two blocks that
// changed are re-reduced with one 32-wide shared-memory read each.  A pop
// costs a fixed handful of warp reductions whatever the budget (up to 64
// blocks, 2048 slots), instead of a per-lane rescan that grew with B.
//
// Order keys are 64 bits: the fp32 score's order key, then a tie key that
// packs the tuple's first ranks (exactly equal fp32 scores are common with
// bf16 logits: 45-65% of popped prefixes share a score).  Only entries that
// agree on score and on every packed rank fall back to an exact rank-tuple
// comparison that walks parent pointers to the common ancestor.
#pragma once

#include "common.cuh"

namespace ddt {

// Threads of the build CTA: the enumeration's level passes, scans and sorts
// scale with the block; the heap fallback uses one warp either way.
// Measured (one request, L = 16): 256 threads are faster at B = 64 (8.2 vs
// 8.8 us), 512 at B = 256 (27.9 vs 36.1 us) and B = 1024 (110 vs 142 us);
// 1024 threads were slower than 512 at every B.
constexpr int BUILD_THREADS_SMALL = 256;
constexpr int BUILD_THREADS_LARGE = 512;
constexpr int BUILD_LARGE_FROM_B = 129;
inline int build_threads(int B) { return B >= BUILD_LARGE_FROM_B ? BUILD_THREADS_LARGE : BUILD_THREADS_SMALL; }

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

// A frontier entry's 64-bit order key and its slot.
struct Best {
  uint32_t hi, lo;   // score key, tie key; hi == 0: none
  int slot;
};

struct BuildSmem {
  float* lp;         // [L][kc]
  uint2* key;        // [B+1] slot order keys (score key, tie key); (0,0) = empty
  float* sc;         // [B+1] slot score
  float* ps;         // [B+1] score of the slot entry's parent node
  uint32_t* mt;      // [B+1] packed parent/depth/rank
  int* nd_parent;    // [B+1]
  int* nd_rank;
  int* nd_depth;
  float* nd_score;
};

// node arrays (16n bytes), the lp table (padded to 16 bytes), keys (8n), slot score, parent score, metadata (12n)
__host__ __device__ inline size_t build_smem_bytes(int L, int kc, int B) {
  const size_t n = (size_t)B + 1;
  return n * 16 + (((size_t)L * kc * 4 + 15) & ~(size_t)15) + n * (8 + 4 + 4 + 4);
}
__host__ __device__ inline size_t enum_smem_bytes();
// with the enumeration arrays after the heap's
__host__ __device__ inline size_t build_smem_bytes_enum(int L, int kc, int B) {
  return ((build_smem_bytes(L, kc, B) + 15) & ~(size_t)15) + enum_smem_bytes();
}

// a before b in the pop order
__device__ __forceinline__ bool best_before(const Best& a, const Best& b, const BuildSmem& sm) {
  if (a.hi != b.hi) return a.hi > b.hi;
  if (a.lo != b.lo) return a.lo > b.lo;
  return tuple_less(sm.mt[a.slot], sm.mt[b.slot], sm.nd_parent, sm.nd_rank);
}

// The warp-wide best among one candidate per lane (hi == 0: none).  Equal
// keys are rare and resolved by the exact tuple comparison.
__device__ __forceinline__ Best warp_best(const Best& c, const BuildSmem& sm) {
  Best r;
  r.hi = __reduce_max_sync(0xffffffffu, c.hi);
  if (r.hi == 0) { r.lo = 0; r.slot = -1; return r; }
  unsigned eq = __ballot_sync(0xffffffffu, c.hi == r.hi);
  r.lo = c.lo;
  if (eq & (eq - 1)) {
    r.lo = __reduce_max_sync(0xffffffffu, c.hi == r.hi ? c.lo : 0u);
    eq = __ballot_sync(0xffffffffu, c.hi == r.hi && c.lo == r.lo);
  }
  int wl = __ffs(eq) - 1;
  r.slot = __shfl_sync(0xffffffffu, c.slot, wl);
  r.lo = __shfl_sync(0xffffffffu, c.lo, wl);
  eq &= eq - 1;
  while (eq) {                       // identical keys: smallest rank tuple
    const int l2 = __ffs(eq) - 1;
    eq &= eq - 1;
    Best o;
    o.hi = r.hi;
    o.lo = r.lo;
    o.slot = __shfl_sync(0xffffffffu, c.slot, l2);
    if (best_before(o, r, sm)) r = o;
  }
  return r;
}

// Register-resident queue for budgets with at most E slots per lane:
// slot s's order key lives in register s / 32 of lane s % 32 (its score,
// parent score and metadata in shared memory).  A pop is a lane-local best
// over E registers and one warp-wide selection; the popped entry's lane
// takes its next sibling and the child's lane its first child, in
// registers, with no re-reduction.  Returns the number of pops.
template <int E>
__device__ __forceinline__ int heap_registers(const BuildSmem& sm, int L, int B, int kc, TieCode tc, int lane) {
  uint32_t kh[E], kl[E];
#pragma unroll
  for (int e = 0; e < E; ++e) { kh[e] = 0u; kl[e] = 0u; }
  int next_slot = 0;
  if (B > 0) {
    const float s0 = __fadd_rn(0.f, sm.lp[0]);
    if (lane == 0) {
      kh[0] = score_key(s0);
      kl[0] = ~tc.unit(1);
      sm.sc[0] = s0;
      sm.ps[0] = 0.f;
      sm.mt[0] = pack_meta(0, 1, 0);
    }
    next_slot = 1;
  }
  __syncwarp();
  int pops = 0;
  while (pops < B) {
    Best lb{0u, 0u, -1};
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const Best c{kh[e], kl[e], lane + 32 * e};
      if (c.hi != 0 && (lb.hi == 0 || best_before(c, lb, sm))) lb = c;
    }
    const Best top = warp_best(lb, sm);
    if (top.hi == 0) break;   // frontier empty
    const int slot = top.slot;
    const uint32_t meta = sm.mt[slot];
    const float sc = sm.sc[slot], ps = sm.ps[slot];
    const uint32_t packed = ~top.lo;
    const int par = meta_parent(meta), d = meta_depth(meta), rk = meta_rank(meta);
    const int node = ++pops;
    const bool sib = rk + 1 < kc;              // next sibling: same parent, next rank
    const bool child = d < L;                  // first child: one position deeper
    const float lsib = sib ? sm.lp[(d - 1) * kc + rk + 1] : 0.f;
    const float lchild = child ? sm.lp[d * kc] : 0.f;
    const float ssib = __fadd_rn(ps, lsib);
    const float schild = __fadd_rn(sc, lchild);
    const int cslot = next_slot;
    __syncwarp();
    if (lane == 0) {
      sm.nd_parent[node] = par;
      sm.nd_rank[node] = rk;
      sm.nd_depth[node] = d;
      sm.nd_score[node] = sc;
      sm.sc[slot] = ssib;
      sm.ps[slot] = ps;
      sm.mt[slot] = pack_meta(par, d, rk + 1);
      if (child) {
        sm.sc[cslot] = schild;
        sm.ps[cslot] = sc;
        sm.mt[cslot] = pack_meta(node, d + 1, 0);
      }
    }
    const uint32_t ksh = sib ? score_key(ssib) : 0u, ksl = sib ? ~(packed + tc.unit(d)) : 0u;
    const uint32_t kch = score_key(schild), kcl = ~(packed + tc.unit(d + 1));
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (slot == lane + 32 * e) { kh[e] = ksh; kl[e] = ksl; }
      if (child && cslot == lane + 32 * e) { kh[e] = kch; kl[e] = kcl; }
    }
    if (child) ++next_slot;
    __syncwarp();
  }
  return pops;
}

// Tournament queue for large budgets (see the file comment).  Returns the
// number of pops.
__device__ __forceinline__ int heap_tournament(const BuildSmem& sm, int L, int B, int kc, TieCode tc, int lane) {
  // cached best of blocks `lane` and `lane + 32`
  Best b0{0u, 0u, -1}, b1{0u, 0u, -1};
  int next_slot = 0;
  if (B > 0) {   // the frontier starts with the best token of position 1
    const float s0 = __fadd_rn(0.f, sm.lp[0]);
    const uint32_t k0 = score_key(s0), t0 = ~tc.unit(1);
    if (lane == 0) {
      sm.key[0] = make_uint2(k0, t0);
      sm.sc[0] = s0;
      sm.ps[0] = 0.f;
      sm.mt[0] = pack_meta(0, 1, 0);
      b0 = Best{k0, t0, 0};
    }
    next_slot = 1;
  }
  __syncwarp();
  // re-reduce block `blk` from shared memory into its owner's cached best
  auto refresh = [&](int blk) {
    const int s = 32 * blk + lane;
    Best c{0u, 0u, -1};
    if (s < next_slot) {
      const uint2 k = sm.key[s];
      c = Best{k.x, k.y, s};
    }
    const Best w = warp_best(c, sm);
    if (lane == (blk & 31)) {
      if (blk < 32) b0 = w;
      else b1 = w;
    }
  };
  int pops = 0;
  while (pops < B) {
    const Best lb = (b1.hi != 0 && (b0.hi == 0 || best_before(b1, b0, sm))) ? b1 : b0;
    const Best top = warp_best(lb, sm);
    if (top.hi == 0) break;   // frontier empty
    const int slot = top.slot;
    const uint32_t meta = sm.mt[slot];
    const float sc = sm.sc[slot], ps = sm.ps[slot];
    const uint32_t packed = ~top.lo;                     // the popped entry's packed ranks
    const int par = meta_parent(meta), d = meta_depth(meta), rk = meta_rank(meta);
    const int node = ++pops;
    const bool sib = rk + 1 < kc;              // next sibling: same parent, next rank
    const bool child = d < L;                  // first child: one position deeper
    const float lsib = sib ? sm.lp[(d - 1) * kc + rk + 1] : 0.f;
    const float lchild = child ? sm.lp[d * kc] : 0.f;
    const float ssib = __fadd_rn(ps, lsib);
    const float schild = __fadd_rn(sc, lchild);
    const int cslot = next_slot;
    __syncwarp();
    if (lane == 0) {
      sm.nd_parent[node] = par;
      sm.nd_rank[node] = rk;
      sm.nd_depth[node] = d;
      sm.nd_score[node] = sc;
      sm.key[slot] = sib ? make_uint2(score_key(ssib), ~(packed + tc.unit(d))) : make_uint2(0u, 0u);
      sm.sc[slot] = ssib;
      sm.ps[slot] = ps;
      sm.mt[slot] = pack_meta(par, d, rk + 1);
      if (child) {
        sm.key[cslot] = make_uint2(score_key(schild), ~(packed + tc.unit(d + 1)));
        sm.sc[cslot] = schild;
        sm.ps[cslot] = sc;
        sm.mt[cslot] = pack_meta(node, d + 1, 0);
      }
    }
    if (child) ++next_slot;
    __syncwarp();
    refresh(slot >> 5);
    if (child && (cslot >> 5) != (slot >> 5)) refresh(cslot >> 5);
  }
  return pops;
}


// ---------------------------------------------------------------------------
// Threshold enumeration (all threads of the CTA).
//
// The heap pops prefixes in one total order: score descending, then rank
// tuple ascending.  A child never precedes its parent (lp <= 0 and fp32
// addition is monotone) and a next sibling never precedes its elder sibling
// (lp sorted within a position), so the first B pops are exactly the B
// largest prefixes of that order, in order.  This path finds them without
// popping one at a time:
//  1. A score threshold t that at least B prefixes reach: the B-th largest
//     score among the prefixes (0,...,0,r) -- greedy chain, one deviation at
//     the last position -- which are real prefixes with their exact scores.
//  2. Every prefix scoring >= t, one depth level per step: a node's children
//     that qualify are the ranks 0..c-1 (scores fall with the rank), c found
//     by binary search; a block scan places them.  Prefix-closed by (1).
//  3. Order the enumerated set by (score, tuple): 64-bit keys (score key,
//     packed leading ranks) with an exact tuple walk on equal keys; the first
//     B entries are the pops.
// If the set exceeds ENUM_CAP entries the caller runs the heap instead.
// ---------------------------------------------------------------------------
constexpr int ENUM_CAP = 4096;
constexpr uint32_t ENUM_ROOT = 0x1FFFu;        // parent field of depth-1 entries

__device__ __forceinline__ uint32_t e_pack(uint32_t parent, int depth, int rank) {
  return parent | ((uint32_t)depth << 13) | ((uint32_t)rank << 19);
}
__device__ __forceinline__ uint32_t e_parent(uint32_t m) { return m & 0x1FFFu; }
__device__ __forceinline__ int e_depth(uint32_t m) { return (int)((m >> 13) & 0x3Fu); }
__device__ __forceinline__ int e_rank(uint32_t m) { return (int)(m >> 19); }

struct EnumSmem {
  float* score;                 // [ENUM_CAP]
  uint32_t* meta;               // [ENUM_CAP] parent entry, depth, rank
  unsigned long long* key;      // [ENUM_CAP] score key << 32 | tie key
  int* off;                     // [ENUM_CAP + 1] per-level child counts -> offsets
  uint16_t* ord;                // [ENUM_CAP] sorted entry indices
  uint16_t* pos;                // [ENUM_CAP] node index of an entry (0: not selected)
};

__host__ __device__ inline size_t enum_smem_bytes() { return (size_t)ENUM_CAP * (4 + 4 + 8 + 2 + 2) + (ENUM_CAP + 1) * 4; }

// Lexicographic tuple comparison of two enumerated entries (a proper prefix
// is smaller): lift the deeper entry, then walk both up to a common parent.
__device__ __forceinline__ bool e_tuple_less(int a, int b, const uint32_t* meta) {
  uint32_t ma = meta[a], mb = meta[b];
  int da = e_depth(ma), db = e_depth(mb);
  int ra = e_rank(ma), rb = e_rank(mb);
  uint32_t pa = e_parent(ma), pb = e_parent(mb);
  const bool a_shorter = da < db;
  while (da > db) { ma = meta[pa]; ra = e_rank(ma); pa = e_parent(ma); --da; }
  while (db > da) { mb = meta[pb]; rb = e_rank(mb); pb = e_parent(mb); --db; }
  if (pa == pb && ra == rb) return a_shorter;
  while (pa != pb) {
    ma = meta[pa]; ra = e_rank(ma); pa = e_parent(ma);
    mb = meta[pb]; rb = e_rank(mb); pb = e_parent(mb);
  }
  return ra < rb;
}

// entry a pops before entry b
__device__ __forceinline__ bool e_before(int a, int b, const EnumSmem& es) {
  const unsigned long long ka = es.key[a], kb = es.key[b];
  if (ka != kb) return ka > kb;
  return e_tuple_less(a, b, es.meta);
}

// In-place exclusive scan of v[0..m) by the whole block; returns the total.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int* v, int m, int* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int per = (m + NT - 1) / NT;
  const int b0 = tid * per, b1 = min(m, b0 + per);
  int sum = 0;
  for (int i = b0; i < b1; ++i) sum += v[i];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int t = warp_tot[w];
    if (w < wid) wbase += t;
    total += t;
  }
  int run = wbase + incl - sum;
  for (int i = b0; i < b1; ++i) {
    const int c = v[i];
    v[i] = run;
    run += c;
  }
  __syncthreads();
  return total;
}

// Returns the number of pops, or -1 when the enumeration exceeds ENUM_CAP.
// Block-uniform.  Fills sm.nd_* for nodes 1..pops.
// kfloor > 0 raises the score threshold: only prefixes whose score key is
// at least kfloor are listed (the adaptive budget's floor).
template <int NT>
__device__ int enum_build(const BuildSmem& sm, const EnumSmem& es, int L, int B, int kc, TieCode tc,
                          uint32_t* hist, int* bcast, int* warp_tot, float* chain, int* s_lev, uint32_t kfloor) {
  const int tid = threadIdx.x;
  // ---- 1. threshold: B-th best score among the one-deviation chain prefixes ----
  if (tid == 0) {
    float c = 0.f;
    for (int d = 0; d < L; ++d) {
      chain[d] = c;                               // score of (0,...,0) of length d
      c = __fadd_rn(c, sm.lp[d * kc]);
    }
  }
  __syncthreads();
  uint32_t t = 1u;                                // every finite or -inf score
  if ((long long)L * kc >= B) {
    // One histogram over the family's key range [kmin, kmax] in 256 equal
    // bins; the lower edge of the bin where the count from the top reaches B
    // is a threshold that at least B prefixes reach (a lower bound of the
    // B-th best, within one bin).  The largest family score is lp[0][0]
    // (chains only fall); the smallest is the last rank at some depth.
    const uint32_t kmax = score_key(sm.lp[0]);
    if (tid < 32) {
      uint32_t kmin = 0xFFFFFFFFu;
      for (int d = tid; d < L; d += 32) kmin = min(kmin, score_key(__fadd_rn(chain[d], sm.lp[d * kc + kc - 1])));
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      if (tid == 0) bcast[0] = (int)kmin;
    }
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    const uint32_t kmin = (uint32_t)bcast[0];
    int shift = 0;
    while (((kmax - kmin) >> shift) >= 256u) ++shift;
    for (int i = tid; i < L * kc; i += NT) {
      const int d = i / kc;
      const uint32_t key = score_key(__fadd_rn(chain[d], sm.lp[i]));
      atomicAdd(&hist[(key - kmin) >> shift], 1u);
    }
    __syncthreads();
    if (tid < 32) {   // lane l holds bins 255-8l .. 248-8l (descending)
      uint32_t c[8];
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[255 - 8 * tid - j]; mine += c[j]; }
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t before = incl - mine;
      const unsigned m = __ballot_sync(0xffffffffu, before < (uint32_t)B && (uint32_t)B <= incl);
      if (tid == __ffs(m) - 1) {
        uint32_t acc = before;
        int jb = 7;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc += c[j];
          if (acc >= (uint32_t)B) { jb = j; break; }
        }
        bcast[1] = 255 - 8 * tid - jb;
      }
      if (m == 0 && tid == 0) bcast[1] = 0;        // cannot happen (L*kc >= B); keep every key
    }
    __syncthreads();
    t = kmin + ((uint32_t)bcast[1] << shift);
    if (t == 0u) t = 1u;
  }
  if (kfloor > t) t = kfloor;
  // ---- 2. every prefix with score key >= t, level by level ----
  // depth 1: children of the root
  if (tid == 0) {
    int lo = 0, hi = kc;                          // first rank failing the threshold
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (score_key(sm.lp[mid]) >= t) lo = mid + 1; else hi = mid;
    }
    s_lev[0] = 0;
    s_lev[1] = lo;
    s_lev[2] = lo > ENUM_CAP ? 1 : 0;
  }
  __syncthreads();
  if (s_lev[2]) return -1;
  int ls = 0, le = s_lev[1];
  for (int r = tid; r < le; r += NT) {
    const float sc = __fadd_rn(0.f, sm.lp[r]);
    es.score[r] = sc;
    es.meta[r] = e_pack(ENUM_ROOT, 1, r);
    const uint32_t code = (uint32_t)(r + 1) * tc.unit(1);
    es.key[r] = ((unsigned long long)score_key(sc) << 32) | (uint32_t)~code;
  }
  __syncthreads();
  for (int d = 1; d < L && le > ls; ++d) {        // parents at depth d, children at depth d+1
    const int m = le - ls;
    const float* lpd = sm.lp + d * kc;
    for (int i = tid; i < m; i += NT) {
      const float ps = es.score[ls + i];
      int lo = 0, hi = kc;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (score_key(__fadd_rn(ps, lpd[mid])) >= t) lo = mid + 1; else hi = mid;
      }
      es.off[i] = lo;
    }
    __syncthreads();
    const int T = block_exclusive_scan<NT>(es.off, m, warp_tot);
    if (le + T > ENUM_CAP) return -1;             // block-uniform
    if (tid == 0) es.off[m] = T;
    __syncthreads();
    const uint32_t unit = tc.unit(d + 1);
    for (int j = tid; j < T; j += NT) {
      int lo = 0, hi = m;                         // last parent with off <= j
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (es.off[mid] <= j) lo = mid; else hi = mid;
      }
      const int par = ls + lo;
      const int r = j - es.off[lo];
      const float sc = __fadd_rn(es.score[par], lpd[r]);
      const int e = le + j;
      es.score[e] = sc;
      es.meta[e] = e_pack((uint32_t)par, d + 1, r);
      const uint32_t code = ~(uint32_t)es.key[par] + (uint32_t)(r + 1) * unit;
      es.key[e] = ((unsigned long long)score_key(sc) << 32) | (uint32_t)~code;
    }
    __syncthreads();
    ls = le;
    le += T;
  }
  // ---- 3. order: position of every entry among the enumerated set ----
  const int total = le;
  const int npop = total < B ? total : B;
  if (total <= NT) {
    // rank by counting; g threads share one entry
    int g = 32;
    while (g > 1 && total * g > NT) g >>= 1;
    const int q = tid / g, part = tid - q * g;
    int rank = 0;
    if (q < total) {
      // 64-bit keys first (four independent counts); equal keys (identical
      // score and leading ranks) are settled by the tuple walk
      const unsigned long long kq = es.key[q];
      int r0 = 0, r1 = 0, r2 = 0, r3 = 0, ties = 0;
      int j = part;
      for (; j + 3 * g < total; j += 4 * g) {
        const unsigned long long k0 = es.key[j], k1 = es.key[j + g], k2 = es.key[j + 2 * g], k3 = es.key[j + 3 * g];
        r0 += k0 > kq; r1 += k1 > kq; r2 += k2 > kq; r3 += k3 > kq;
        ties += (k0 == kq) + (k1 == kq) + (k2 == kq) + (k3 == kq);
      }
      for (; j < total; j += g) {
        const unsigned long long kj = es.key[j];
        r0 += kj > kq;
        ties += kj == kq;
      }
      rank = (r0 + r1) + (r2 + r3);
      if (ties > (part == (q % g) ? 1 : 0))       // another entry shares the key
        for (int jj = part; jj < total; jj += g)
          if (jj != q && es.key[jj] == kq && e_tuple_less(jj, q, es.meta)) ++rank;
    }
    for (int o = g >> 1; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (q < total && part == 0) es.pos[q] = (uint16_t)(rank < npop ? rank + 1 : 0);
  } else {
    int P = 1;
    while (P < total) P <<= 1;
    for (int i = tid; i < P; i += NT) es.ord[i] = (uint16_t)(i < total ? i : 0xFFFFu);
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        // up to four compare-exchanges per thread, their loads issued together
        for (int i0 = tid; i0 < P / 2; i0 += 4 * NT) {
          int lo[4], hi[4];
          uint16_t a[4], b[4];
          unsigned long long ka[4], kb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * NT;
            lo[u] = 2 * stride * (i / stride) + (i % stride);
            hi[u] = lo[u] + stride;
            const bool in = i < P / 2;
            a[u] = in ? es.ord[lo[u]] : 0xFFFFu;
            b[u] = in ? es.ord[hi[u]] : 0xFFFFu;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ka[u] = a[u] != 0xFFFFu ? es.key[a[u]] : 0ull;
            kb[u] = b[u] != 0xFFFFu ? es.key[b[u]] : 0ull;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (i0 + u * NT >= P / 2) continue;
            const bool up = (lo[u] & size) == 0;   // this run sorts in pop order
            // b before a (pads last)
            bool b_first;
            if (b[u] == 0xFFFFu) b_first = false;
            else if (a[u] == 0xFFFFu) b_first = true;
            else if (ka[u] != kb[u]) b_first = kb[u] > ka[u];
            else b_first = e_tuple_less(b[u], a[u], es.meta);
            if (b_first == up) { es.ord[lo[u]] = b[u]; es.ord[hi[u]] = a[u]; }
          }
        }
        __syncthreads();
      }
    }
    for (int i = tid; i < total; i += NT) es.pos[i] = 0;
    __syncthreads();
    for (int i = tid; i < npop; i += NT) es.pos[es.ord[i]] = (uint16_t)(i + 1);
  }
  __syncthreads();
  // ---- nodes 1..npop in pop order ----
  for (int e = tid; e < total; e += NT) {
    const int node = es.pos[e];
    if (node == 0) continue;
    const uint32_t mt = es.meta[e];
    const uint32_t pe = e_parent(mt);
    sm.nd_parent[node] = pe == ENUM_ROOT ? 0 : (int)es.pos[pe];
    sm.nd_rank[node] = e_rank(mt);
    sm.nd_depth[node] = e_depth(mt);
    sm.nd_score[node] = es.score[e];
  }
  return npop;
}

template <int NT>
__global__ void __launch_bounds__(NT, 1)
build_kernel(const int32_t* __restrict__ ids, const float* __restrict__ lp,
             const int32_t* __restrict__ root_token, int L, int K, int B, int kc, TieCode tc, int use_enum,
             const float* __restrict__ gain_floor, int32_t* __restrict__ node_token, int32_t* __restrict__ parent,
             int32_t* __restrict__ depth, int32_t* __restrict__ node_rank,
             float* __restrict__ score, uint32_t* __restrict__ anc, int32_t* __restrict__ n_nodes,
             int32_t* __restrict__ build_path) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int r = blockIdx.x;
  const int tid = threadIdx.x;
  const int n = B + 1;
  const int W = (n + 31) >> 5;
  // the round's attention may start its prefix tiles now (it waits for this
  // grid before reading the tree)
  griddep_launch_dependents();

  BuildSmem sm;
  {
    // the node arrays first: everything after them is dead once the pops are known
    unsigned char* p = smem_raw;
    sm.nd_parent = (int*)p; p += (size_t)n * 4;
    sm.nd_rank = (int*)p;   p += (size_t)n * 4;
    sm.nd_depth = (int*)p;  p += (size_t)n * 4;
    sm.nd_score = (float*)p; p += (size_t)n * 4;
    sm.lp = (float*)p;      p += ((size_t)L * kc * 4 + 15) & ~(size_t)15;   // 16-byte aligned
    sm.key = (uint2*)p;     p += (size_t)n * 8;
    sm.sc = (float*)p;      p += (size_t)n * 4;
    sm.ps = (float*)p;      p += (size_t)n * 4;
    sm.mt = (uint32_t*)p;
  }
  EnumSmem es;
  {
    unsigned char* p = smem_raw + ((build_smem_bytes(L, kc, B) + 15) & ~(size_t)15);
    es.key = (unsigned long long*)p; p += (size_t)ENUM_CAP * 8;
    es.score = (float*)p;            p += (size_t)ENUM_CAP * 4;
    es.meta = (uint32_t*)p;          p += (size_t)ENUM_CAP * 4;
    es.off = (int*)p;                p += (size_t)(ENUM_CAP + 1) * 4;
    es.ord = (uint16_t*)p;           p += (size_t)ENUM_CAP * 2;
    es.pos = (uint16_t*)p;
  }
  __shared__ int s_pops;
  __shared__ uint32_t s_hist[256];
  __shared__ int s_bcast[4];
  __shared__ int s_warp_tot[NT / 32];
  __shared__ float s_chain[64];
  __shared__ int s_lev[3];

  // stage the lp table (only ranks < kc can ever be popped)
  const float* lpr = lp + (size_t)r * L * K;
  if ((kc & 3) == 0 && (K & 3) == 0 && ((uintptr_t)lpr & 15) == 0) {
    // 16-byte loads, all of a thread's issued before any is stored
    const int q4 = kc >> 2, total4 = L * q4;
    for (int i0 = tid; i0 < total4; i0 += 4 * NT) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * NT;
        const int d = i / q4, k4 = i - d * q4;
        if (i < total4) v[u] = *reinterpret_cast<const float4*>(lpr + (size_t)d * K + 4 * k4);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * NT;
        if (i < total4) reinterpret_cast<float4*>(sm.lp)[i] = v[u];
      }
    }
  } else {
    for (int i = tid; i < L * kc; i += NT) {
      const int d = i / kc, k = i - d * kc;
      sm.lp[i] = lpr[(size_t)d * K + k];
    }
  }
  __syncthreads();

  if (tid == 0) {
    sm.nd_parent[0] = -1;
    sm.nd_rank[0] = -1;
    sm.nd_depth[0] = 0;
    sm.nd_score[0] = 0.f;
  }
  // Adaptive budget: only pops whose score exceeds the request's floor are
  // kept (NaN keeps nothing).  Pops come in non-increasing score order, so
  // the kept ones are a leading run of the pop sequence.
  float floor_v = -INFINITY;
  bool has_floor = false;
  if (gain_floor != nullptr) {
    floor_v = gain_floor[r];
    if (floor_v != floor_v) floor_v = INFINITY;
    has_floor = true;
  }
  // the smallest order key above the floor (scores compare by their keys)
  const uint32_t kfloor = !has_floor ? 0u : (floor_v == INFINITY ? 0xFFFFFFFFu : score_key(floor_v) + 1u);
  int epops = -1, how = 0;
  if (use_enum && B > 0)
    epops = enum_build<NT>(sm, es, L, B, kc, tc, s_hist, s_bcast, s_warp_tot, s_chain, s_lev, kfloor);
  if (epops >= 0) {
    if (tid == 0) s_pops = epops;
  } else if (B > 0) {
    how = n <= 32 * 3 ? 1 : (n <= 32 * 9 ? 2 : 3);
    if (tid < 32) {
      const int lane = tid;
      int pops;
      if (how == 1) pops = heap_registers<3>(sm, L, B, kc, tc, lane);
      else if (how == 2) pops = heap_registers<9>(sm, L, B, kc, tc, lane);
      else pops = heap_tournament(sm, L, B, kc, tc, lane);
      if (lane == 0) s_pops = pops;
    }
  } else if (tid == 0) {
    s_pops = 0;
  }
  __syncthreads();
  if (has_floor) {
    // count of the leading pops above the floor
    __shared__ int s_keep;
    if (tid == 0) s_keep = 0;
    __syncthreads();
    const int pops = s_pops;
    int keep = 0;
    for (int i = 1 + tid; i <= pops; i += NT) keep += score_key(sm.nd_score[i]) >= kfloor ? 1 : 0;
    keep = __reduce_add_sync(0xffffffffu, keep);
    if ((tid & 31) == 0 && keep) atomicAdd(&s_keep, keep);
    __syncthreads();
    if (tid == 0) s_pops = s_keep;
    __syncthreads();
  }
  if (build_path != nullptr && tid == 0) build_path[r] = how;

  // ---- outputs ----
  const int nn = s_pops + 1;
  const size_t ro = (size_t)r * n;
  const int32_t* idr = ids + (size_t)r * L * K;
  // Ancestor rows for wide masks: built in shared memory one depth level at a
  // time (row i = row parent(i) | bit i, a warp per row, lanes over words),
  // then written out with 16-byte stores.  Needs n*W words of the dead area.
  const size_t dead = (use_enum ? build_smem_bytes_enum(L, kc, B) : build_smem_bytes(L, kc, B)) - (size_t)n * 16;
  const bool smem_rows = W >= 4 && (size_t)n * (W + 1) * 4 <= dead;
  if (smem_rows) {
    uint32_t* rows = reinterpret_cast<uint32_t*>(smem_raw + (size_t)n * 16);   // [n][W]
    int* order = reinterpret_cast<int*>(rows + (size_t)n * W);                  // [n] nodes sorted by depth
    __shared__ int s_dcnt[66];
    for (int i = tid; i < 66; i += NT) s_dcnt[i] = 0;
    __syncthreads();
    for (int i = tid; i < nn; i += NT) atomicAdd(&s_dcnt[sm.nd_depth[i] + 1], 1);
    __syncthreads();
    if (tid == 0)
      for (int d = 1; d < 66; ++d) s_dcnt[d] += s_dcnt[d - 1];   // s_dcnt[d]: first slot of depth d
    __syncthreads();
    for (int i = tid; i < nn; i += NT) order[atomicAdd(&s_dcnt[sm.nd_depth[i]], 1)] = i;
    __syncthreads();
    // after the scatter s_dcnt[d] is the end of depth d: depth d spans [s_dcnt[d-1], s_dcnt[d])
    const int lane = tid & 31, wrp = tid >> 5;
    for (int w = lane; w < W; w += 32) rows[w] = (w == 0) ? 1u : 0u;   // the root row
    __syncthreads();
    for (int d = 1; d <= L; ++d) {
      const int b0 = s_dcnt[d - 1], b1 = s_dcnt[d];
      if (b0 >= b1) break;
      for (int k = b0 + wrp; k < b1; k += NT / 32) {
        const int i = order[k];
        const int pi = sm.nd_parent[i];
        if (!DDT_IN_RANGE(pi, 0, i)) continue;
        for (int w = lane; w < W; w += 32)
          rows[(size_t)i * W + w] = rows[(size_t)pi * W + w] | ((i >> 5) == w ? (1u << (i & 31)) : 0u);
      }
      __syncthreads();
    }
    for (int i = nn * W + tid; i < n * W; i += NT) rows[i] = 0u;   // absent nodes
    __syncthreads();
    uint32_t* arow0 = anc + ro * W;
    const int words = n * W;
    if (((uintptr_t)arow0 & 15) == 0) {
      for (int i = tid; i < words / 4; i += NT)
        reinterpret_cast<uint4*>(arow0)[i] = reinterpret_cast<const uint4*>(rows)[i];
      for (int i = (words & ~3) + tid; i < words; i += NT) arow0[i] = rows[i];
    } else {
      for (int i = tid; i < words; i += NT) arow0[i] = rows[i];
    }
  }
  for (int i = tid; i < n; i += NT) {
    bool live = i < nn;
    if (live && i > 0)   // a live node's parent precedes it, its depth is a block position, its rank a top-K rank
      live = DDT_IN_RANGE(sm.nd_parent[i], 0, i) && DDT_IN_RANGE(sm.nd_depth[i], 1, L + 1) &&
             DDT_IN_RANGE(sm.nd_rank[i], 0, kc);
    const int d = live ? sm.nd_depth[i] : -1;
    const int rk = live ? sm.nd_rank[i] : -1;
    if (node_token) node_token[ro + i] = !live ? -1 : (i == 0 ? root_token[r] : idr[(size_t)(d - 1) * K + rk]);
    parent[ro + i] = live ? sm.nd_parent[i] : -1;
    if (depth) depth[ro + i] = d;
    if (node_rank) node_rank[ro + i] = rk;
    if (score) score[ro + i] = live ? sm.nd_score[i] : -INFINITY;
    if (smem_rows) continue;
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
