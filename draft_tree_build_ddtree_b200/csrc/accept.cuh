// Stage 4: greedy verifier walk and in-place KV compaction.
//
// "DDTree Deep Dive" §6 (verifier walk: take the target's argmax at the
// current node, descend into the child carrying that token, the first
// unmatched argmax is the next bonus token) and §5 (only the accepted path's
// KV is kept; tree tokens are interleaved in the cache tail, so the accepted
// rows are compacted in place).
//
// Kernel 1 (argmax): HBM-bound streaming pass over the target logits of the
// live tree nodes.  Rows are cut into chunks so that the grid is about one
// wave of resident 256-thread CTAs; every thread keeps its running best
// (value, lowest index) over batches of 16-byte loads.  Each CTA reduces its
// chunk to one 64-bit composite (order key of the logit, then the
// complemented token id, so lower ids win ties) and merges it with atomicMax
// into the row's workspace slot.  One ticket per request counts its finished
// CTAs; the last one (nobody waits) reads every live row's slot, publishes
// the argmax and resets the slot, and when the walk is fused it loads the
// tree in the same round of loads and runs the request's walk and
// compaction itself.
// Kernel 2 (walk + compaction, for caches with many layers): one CTA per
// (request, layer, K/V).
// The walk: node j is the accepted child of its parent iff its token equals
// the parent's argmax (siblings carry distinct tokens, so at most one child
// matches), giving next[parent] = j in shared memory; the walk follows next[]
// from the root.  Compaction loads every source row of a (layer, K/V) into
// registers before writing any destination, in forward batches (a later
// batch's sources lie above every destination of an earlier batch because
// path[j] >= j).
#pragma once

#include "common.cuh"
#include "topk.cuh"

namespace ddt {

constexpr int ARGMAX_THREADS = 256;
constexpr int ARGMAX_VPT = 10;     // 16-byte loads per thread per batch
constexpr int ARGMAX_CTAS_PER_SM = 4;
constexpr int WALK_THREADS = 256;
constexpr int WALK_VPT = 8;        // 16-byte registers per thread per compaction batch
constexpr int WALK_FUSE_MAX_LAYERS = 2;   // compaction by the argmax kernel up to this many layers
constexpr int WALK_MAX_N = 1025;   // B + 1 <= 1025

struct ArgmaxWs {
  unsigned long long* best;  // [rows] running composite maximum
  int32_t* argmax;           // [rows]
  uint32_t* req_ticket;      // [n_req] CTAs finished
};

inline size_t argmax_ws_bytes(int rows, int n_req) {
  return align256((size_t)rows * 8) + align256((size_t)rows * 4) + align256((size_t)n_req * 4);
}
inline ArgmaxWs argmax_ws_carve(void* ws, int rows) {
  char* b = (char*)ws;
  ArgmaxWs w;
  w.best = (unsigned long long*)b;
  b += align256((size_t)rows * 8);
  w.argmax = (int32_t*)b;
  b += align256((size_t)rows * 4);
  w.req_ticket = (uint32_t*)b;
  return w;
}

struct WalkArgs {
  const int32_t* node_token;
  const int32_t* parent;
  const int32_t* n_nodes;
  const int32_t* prefix_len;
  const int32_t* argmax_ws;   // [n_req][n]
  int n, L;
  // outputs
  int32_t* new_prefix_len;
  int32_t* target_argmax;
  int32_t* path;
  int32_t* accept_len;
  int32_t* next_bonus;
  int32_t* src_slot;
  int32_t* dst_slot;
  // cache
  unsigned char* k_cache;
  unsigned char* v_cache;
  const int32_t* block_table;
  int layers, n_req, paged, s_max, num_blocks, max_blocks;
  int row_bytes;              // Hkv * D * element size
};

struct WalkSmem {
  int* nxt;     // [n]
  int* targ;    // [n] target argmax of every node
  int* par;     // [n] parent
  int* tok;     // [n] token
  int* path;    // [33]
  int* k;
  int* ok;
};

// Request r's tree (parent, token of every node slot) and target argmax in
// shared memory, all with one round of loads; next[] cleared.
__device__ __forceinline__ void walk_load(const WalkArgs& a, int r, const WalkSmem& ws) {
  const size_t ro = (size_t)r * a.n;
  for (int i = threadIdx.x; i < a.n; i += blockDim.x) {
    const int p = __ldcg(a.parent + ro + i);
    const int t = __ldcg(a.node_token + ro + i);
    const int g = __ldcg(a.argmax_ws + ro + i);
    ws.par[i] = p;
    ws.tok[i] = t;
    ws.targ[i] = g;
    ws.nxt[i] = -1;
  }
}

// Walk of request r, then compaction of its (layer, K/V) pairs lk0..lk1-1
// (lk = layer * 2 + (0: K, 1: V)); the pair lk == 0 also writes the walk's
// outputs.  All threads of the CTA call it.
// The tree and argmax are in `ws` (walk_load, or the argmax kernel's last
// CTA), followed by a barrier; nn live nodes, committed prefix P.
__device__ void walk_request(const WalkArgs& a, int r, int nn, int P, int lk0, int lk1, const WalkSmem& ws) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const size_t ro = (size_t)r * a.n;
  for (int j = 1 + tid; j < nn; j += nth) {
    const int p = ws.par[j];
    if (p >= 0 && p < j && ws.tok[j] == ws.targ[p]) ws.nxt[p] = j;
  }
  __syncthreads();
  if (tid == 0) {
    int cur = 0, k = 0;
    ws.path[0] = 0;
    while (k < a.L && ws.nxt[cur] >= 0) {
      if (!DDT_IN_RANGE(ws.nxt[cur], cur + 1, nn)) break;
      cur = ws.nxt[cur];
      ws.path[++k] = cur;
    }
    *ws.k = k;
    const long long cap = a.paged ? (long long)a.max_blocks * DDTREE_PAGE : (long long)a.s_max;
    *ws.ok = (P >= 0 && (long long)P + nn <= cap) ? 1 : 0;
  }
  __syncthreads();
  if (a.paged && a.k_cache != nullptr && *ws.ok) {   // blocks holding slots [0, P + nn) must be pool blocks
    const int nb = (P + nn + DDTREE_PAGE - 1) / DDTREE_PAGE;
    int bad = 0;
    for (int b = tid; b < nb; b += nth) {
      const int blk = a.block_table[(size_t)r * a.max_blocks + b];
      bad |= (blk < 0 || blk >= a.num_blocks);
    }
    bad = __syncthreads_or(bad);
    if (tid == 0 && bad) *ws.ok = 0;
    __syncthreads();
  }
  const int k = *ws.k;
  const int ok = *ws.ok;
  if (lk0 == 0) {
    for (int i = tid; i <= a.L; i += nth) {
      const bool on = i <= k;
      if (a.path) a.path[(size_t)r * (a.L + 1) + i] = on ? ws.path[i] : -1;
      if (a.src_slot) a.src_slot[(size_t)r * (a.L + 1) + i] = on ? P + ws.path[i] : -1;
      if (a.dst_slot) a.dst_slot[(size_t)r * (a.L + 1) + i] = on ? P + i : -1;
    }
    if (a.target_argmax)
      for (int i = tid; i < a.n; i += nth) a.target_argmax[ro + i] = i < nn ? ws.targ[i] : -1;
    if (tid == 0) {
      if (a.accept_len) a.accept_len[r] = k + 1;
      if (a.next_bonus) a.next_bonus[r] = ws.targ[ws.path[k]];
      a.new_prefix_len[r] = P + k + 1;
      if (!ok && a.k_cache) flag_status(DDTREE_STATUS_CAPACITY);
    }
  }
  if (a.k_cache == nullptr || !ok || k == 0) return;   // block-uniform

  // ---- compaction: rows j = 1..k move (row 0 is the root, already in place) ----
  const int vec_per_row = a.row_bytes / 16;
  const int total = k * vec_per_row;
  const int per_batch = nth * WALK_VPT;
  for (int lk = lk0; lk < lk1; ++lk) {
    const int layer = lk >> 1;
    unsigned char* cache = (lk & 1) ? a.v_cache : a.k_cache;
    auto row_ptr = [&](int slot) -> unsigned char* {
      size_t rowi;
      if (a.paged) {
        const int blk = a.block_table[(size_t)r * a.max_blocks + slot / DDTREE_PAGE];
        rowi = ((size_t)layer * a.num_blocks + blk) * DDTREE_PAGE + (slot % DDTREE_PAGE);
      } else {
        rowi = ((size_t)layer * a.n_req + r) * a.s_max + slot;
      }
      return cache + rowi * (size_t)a.row_bytes;
    };
    for (int b0 = 0; b0 < total; b0 += per_batch) {
      uint4 buf[WALK_VPT];
#pragma unroll
      for (int t = 0; t < WALK_VPT; ++t) {
        const int e = b0 + t * nth + tid;
        if (e < total) {
          const int j = 1 + e / vec_per_row, c = e % vec_per_row;
          if (DDT_IN_RANGE(ws.path[j], j, nn)) buf[t] = *((const uint4*)row_ptr(P + ws.path[j]) + c);
        }
      }
      __syncthreads();   // every source of this batch is read before any write
#pragma unroll
      for (int t = 0; t < WALK_VPT; ++t) {
        const int e = b0 + t * nth + tid;
        if (e < total) {
          const int j = 1 + e / vec_per_row, c = e % vec_per_row;
          if (ws.path[j] != j && DDT_IN_RANGE(ws.path[j], j, nn)) *((uint4*)row_ptr(P + j) + c) = buf[t];
        }
      }
      __syncthreads();
    }
  }
}

// ---------------------------------------------------------------------------
// Temperature > 0: one draw per tree node from softmax(z / T) by the
// Gumbel-max identity, argmax_v (z_v / T - log(-log u_v)), with u_v from
// Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011): output word v % 4 at counter
// (v / 4, node, request, 0) and key (seed, offset).  The perturbed score is
// formed in fp64 with explicitly rounded operations and rounded once to fp32;
// the argmax then runs exactly as at temperature 0 (lowest id on ties).
// ---------------------------------------------------------------------------
struct SampleArgs {
  double inv_t;                    // 1 / T in fp64
  unsigned long long seed, offset;
};

__device__ __forceinline__ void philox4x64_10(unsigned long long c[4], unsigned long long k0, unsigned long long k1) {
  constexpr unsigned long long M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr unsigned long long W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const unsigned long long hi0 = __umul64hi(M0, c[0]), lo0 = M0 * c[0];
    const unsigned long long hi1 = __umul64hi(M1, c[2]), lo1 = M1 * c[2];
    const unsigned long long n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
    k0 += W0;
    k1 += W1;
  }
}

// The four Philox words of counter (block, node, req, 0).
__device__ __forceinline__ void philox_block(unsigned long long w[4], unsigned long long block, int node, int req,
                                             const SampleArgs& sa) {
  w[0] = block;
  w[1] = (unsigned long long)node;
  w[2] = (unsigned long long)req;
  w[3] = 0ull;
  philox4x64_10(w, sa.seed, sa.offset);
}

// fp32 rounding of z / T + Gumbel(u(word)); u = ((word >> 12) + 1/2) 2^-52 is exact.
__device__ __forceinline__ float gumbel_score(float z, unsigned long long word, double inv_t) {
  const double u = __dmul_rn(__dadd_rn((double)(word >> 12), 0.5), 0x1p-52);
  const double g = -log(-log(u));
  return __double2float_rn(__dadd_rn(__dmul_rn((double)z, inv_t), g));
}

// The argmax of one chunk of a row: per-thread running best over batches of
// 16-byte loads (elements visited in increasing index order, so the first
// maximum -- the lowest index -- is kept; NaN never compares greater and is
// flagged), then a block-wide maximum of 64-bit composites.  SAMPLE: the
// argmax of the Gumbel-perturbed scores (a draw at temperature T > 0).
template <int DT, bool SAMPLE>
__global__ void __launch_bounds__(ARGMAX_THREADS, SAMPLE ? 2 : ARGMAX_CTAS_PER_SM)
argmax_kernel(const void* __restrict__ logits, int n, int V, long long row_stride,
              const int32_t* __restrict__ n_nodes, int cpr, int chunk, ArgmaxWs ws, WalkArgs wa, int fuse_walk,
              SampleArgs sa) {
  constexpr int EPV = (DT == DDTREE_BF16) ? 8 : 4;
  __shared__ unsigned long long red[ARGMAX_THREADS / 32];
  __shared__ int s_last;
  __shared__ int s_nxt[WALK_MAX_N];
  __shared__ int s_targ[WALK_MAX_N];
  __shared__ int s_par[WALK_MAX_N];
  __shared__ int s_tok[WALK_MAX_N];
  __shared__ int s_path[33];
  __shared__ int s_k, s_ok;
  const int tid = threadIdx.x;
  const int row = blockIdx.x / cpr;              // row = req * n + node
  const int c = blockIdx.x - row * cpr;
  const int req = row / n, node = row - req * n;
  const int live = min(n_nodes[req], n);
  if (node >= live) return;                      // absent node: nothing to read
  const long long c0 = (long long)c * chunk;
  const int len = (int)min((long long)chunk, (long long)V - c0);
  const unsigned char* base =
      (const unsigned char*)logits + ((long long)row * row_stride + c0) * (16 / EPV);
  const int nvec_full = len / EPV;

  float bv = -INFINITY;
  uint32_t bi = 0xFFFFFFFFu;                     // chunk-local index of the best; none yet
  uint32_t mag = 0;                              // NaN detection (bf16: both halves)
  auto visit = [&](float f, uint32_t idx) {
    if (f > bv || (bi == 0xFFFFFFFFu && f == bv)) { bv = f; bi = idx; }
  };
  constexpr int VPT = SAMPLE ? 2 : ARGMAX_VPT;     // sampling is compute-bound: fewer loads in flight
  for (int vb = 0; vb < nvec_full; vb += ARGMAX_THREADS * VPT) {
    uint4 vec[VPT];
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int vi = vb + v * ARGMAX_THREADS + tid;
      vec[v] = vi < nvec_full ? ldg_stream_v4(base + (size_t)vi * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int vi = vb + v * ARGMAX_THREADS + tid;
      if (vi < nvec_full) {
        if (!SAMPLE) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t w = u32_at(vec[v], q);
            if (DT == DDTREE_BF16) {
              mag = max(mag, max(w & 0x7FFFu, (w >> 16) & 0x7FFFu));
              visit(__uint_as_float(w << 16), (uint32_t)(vi * EPV + 2 * q));
              visit(__uint_as_float(w & 0xFFFF0000u), (uint32_t)(vi * EPV + 2 * q + 1));
            } else {
              const float f = __uint_as_float(w);
              mag |= (f != f) ? 0xFFFFu : 0u;
              visit(f, (uint32_t)(vi * EPV + q));
            }
          }
        } else {
          // the vector's elements start at a multiple of 4 of the row (chunks are multiples of 8)
          const long long e0 = c0 + (long long)vi * EPV;
#pragma unroll
          for (int b = 0; b < EPV / 4; ++b) {
            unsigned long long rw[4];
            philox_block(rw, (unsigned long long)(e0 / 4 + b), node, req, sa);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = 4 * b + j;
              float f;
              if (DT == DDTREE_BF16) {
                const uint32_t bits = (u32_at(vec[v], e >> 1) >> (16 * (e & 1))) & 0xFFFFu;
                mag = max(mag, bits & 0x7FFFu);
                f = bf16_bits_to_f32((uint16_t)bits);
              } else {
                f = __uint_as_float(u32_at(vec[v], e));
                mag |= (f != f) ? 0xFFFFu : 0u;
              }
              visit(gumbel_score(f, rw[j], sa.inv_t), (uint32_t)(vi * EPV + e));
            }
          }
        }
      }
    }
  }
  // ragged tail of the chunk (V not a multiple of the vector width): one thread, ascending
  if (tid == 0) {
    for (int e = nvec_full * EPV; e < len; ++e) {
      float f;
      if (DT == DDTREE_BF16) {
        const uint32_t bits = ((const uint16_t*)base)[e];
        mag = max(mag, bits & 0x7FFFu);
        f = bf16_bits_to_f32((uint16_t)bits);
      } else {
        f = ((const float*)base)[e];
        mag |= (f != f) ? 0xFFFFu : 0u;
      }
      if (SAMPLE) {
        unsigned long long rw[4];
        const long long g = c0 + e;
        philox_block(rw, (unsigned long long)(g / 4), node, req, sa);
        f = gumbel_score(f, rw[g & 3], sa.inv_t);
      }
      visit(f, (uint32_t)e);
    }
  }
  const bool nan_seen = DT == DDTREE_BF16 ? mag > 0x7F80u : mag != 0u;
  if (__any_sync(0xffffffffu, nan_seen) && (tid & 31) == 0) flag_status(DDTREE_STATUS_NONFINITE);
  unsigned long long best = 0;
  if (bi != 0xFFFFFFFFu) {
    const uint32_t gid = (uint32_t)(c0 + bi);
    best = ((unsigned long long)key32_of_f32(bv) << TOPK_ID_BITS) | (TOPK_ID_MASK - gid);
  }
  best = warp_max_u64(best);
  if ((tid & 31) == 0) red[tid >> 5] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long b = red[0];
    for (int i = 1; i < ARGMAX_THREADS / 32; ++i) b = red[i] > b ? red[i] : b;
    atomicMax(&ws.best[row], b);
    __threadfence();
    const unsigned t = atomicAdd(&ws.req_ticket[req], 1u);
    s_last = (t == (unsigned)(live * cpr - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // The request's last CTA: every live row's argmax (read and reset) and,
  // for the fused walk, the tree, in one round of loads.
  const size_t ro = (size_t)req * n;
  const int P = fuse_walk ? wa.prefix_len[req] : 0;
  for (int i = tid; i < n; i += ARGMAX_THREADS) {
    unsigned long long fin = 0ull;
    int p = -1, tk = -1;
    if (i < live) fin = __ldcg(&ws.best[ro + i]);
    if (fuse_walk) {
      p = __ldcg(wa.parent + ro + i);
      tk = __ldcg(wa.node_token + ro + i);
    }
    if (i < live) {
      // fin == 0: every logit of the row was NaN (flagged); -1 matches no token
      const int32_t am = fin == 0ull ? -1 : (int32_t)(TOPK_ID_MASK - (uint32_t)(fin & TOPK_ID_MASK));
      ws.best[ro + i] = 0ull;
      ws.argmax[ro + i] = am;
      s_targ[i] = am;
    }
    s_par[i] = p;
    s_tok[i] = tk;
    s_nxt[i] = -1;
  }
  if (tid == 0) ws.req_ticket[req] = 0;   // ready for the next call
  if (!fuse_walk) return;
  __syncthreads();
  const WalkSmem sm{s_nxt, s_targ, s_par, s_tok, s_path, &s_k, &s_ok};
  walk_request(wa, req, live, P, 0, wa.k_cache ? 2 * wa.layers : 1, sm);
}

__global__ void __launch_bounds__(WALK_THREADS) walk_compact_kernel(WalkArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];   // [4][n] ints
  __shared__ int s_path[33];
  __shared__ int s_k, s_ok;
  int* sw = (int*)smem_raw;
  const WalkSmem sm{sw, sw + a.n, sw + 2 * a.n, sw + 3 * a.n, s_path, &s_k, &s_ok};
  const int r = blockIdx.x;
  const int nn = min(a.n_nodes[r], a.n);
  const int P = a.prefix_len[r];
  walk_load(a, r, sm);
  __syncthreads();
  walk_request(a, r, nn, P, blockIdx.y, blockIdx.y + 1, sm);
}

}  // namespace ddt
