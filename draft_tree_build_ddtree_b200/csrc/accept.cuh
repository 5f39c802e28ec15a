// Stage 4: greedy verifier walk and in-place KV compaction.
//
// "DDTree Deep Dive" §6 (verifier walk: take the target's argmax at the
// current node, descend into the child carrying that token, the first
// unmatched argmax is the next bonus token) and §5 (only the accepted path's
// KV is kept; tree tokens are interleaved in the cache tail, so the accepted
// rows are compacted in place).
//
// Kernel 1 (argmax): HBM-bound streaming pass over the target logits of the
// live tree nodes, chunked like the top-K stage.  Each CTA reduces its chunk
// to one 64-bit composite (order key of the logit, then the complemented
// token id, so lower ids win ties), merges it with atomicMax into the row's
// workspace slot, and the last CTA of the row (atomic ticket) publishes the
// argmax and resets the slot.
// Kernel 2 (walk + compaction): one CTA per (request, layer, K/V).  Every
// CTA derives the path itself: node j is the accepted child of its parent
// iff its token equals the parent's argmax (siblings carry distinct tokens,
// so at most one child matches), giving next[parent] = j in shared memory;
// the walk then follows next[] from the root.  The CTA loads every source
// row of its (layer, K/V) into registers before writing any destination,
// in forward batches (a later batch's sources lie above every destination
// of an earlier batch because path[j] >= j).
#pragma once

#include "common.cuh"
#include "topk.cuh"

namespace ddt {

constexpr int ARGMAX_THREADS = 512;
constexpr int WALK_THREADS = 256;
constexpr int WALK_VPT = 8;      // 16-byte registers per thread per compaction batch

struct ArgmaxWs {
  unsigned long long* best;  // [rows]
  uint32_t* ticket;          // [rows]
  int32_t* argmax;           // [rows]
};

inline size_t argmax_ws_bytes(int rows) {
  return align256((size_t)rows * 8) + align256((size_t)rows * 4) + align256((size_t)rows * 4);
}
inline ArgmaxWs argmax_ws_carve(void* ws, int rows) {
  char* b = (char*)ws;
  ArgmaxWs w;
  w.best = (unsigned long long*)b;
  b += align256((size_t)rows * 8);
  w.ticket = (uint32_t*)b;
  b += align256((size_t)rows * 4);
  w.argmax = (int32_t*)b;
  return w;
}

// The argmax of one chunk.  bf16: an fp32 max pass (bf16 widens with a
// shift) finds the chunk's largest value, then the threads holding it find
// the lowest index with that value.  fp32: 64-bit (key, complemented id)
// composites.  The chunk winner becomes a 64-bit composite with the global
// token id for the row-wide atomicMax.
template <int DT, int VPT>
__global__ void __launch_bounds__(ARGMAX_THREADS)
argmax_kernel(const void* __restrict__ logits, int n, int V, long long row_stride,
              const int32_t* __restrict__ n_nodes, int cpr, int chunk, ArgmaxWs ws) {
  constexpr int EPV = (DT == DDTREE_BF16) ? 8 : 4;
  __shared__ unsigned long long red[ARGMAX_THREADS / 32];
  __shared__ uint32_t red32[ARGMAX_THREADS / 32];
  __shared__ float redf[ARGMAX_THREADS / 32];
  const int tid = threadIdx.x;
  const int row = blockIdx.x / cpr;              // row = req * n + node
  const int c = blockIdx.x - row * cpr;
  const int req = row / n, node = row - req * n;
  if (node >= n_nodes[req]) return;              // absent node: nothing to read
  const long long c0 = (long long)c * chunk;
  const int len = (int)min((long long)chunk, (long long)V - c0);
  const unsigned char* base =
      (const unsigned char*)logits + ((long long)row * row_stride + c0) * (16 / EPV);
  const int nvec_full = len / EPV;

  uint4 vec[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int vi = v * ARGMAX_THREADS + tid;
    vec[v] = vi < nvec_full ? ldg_stream_v4(base + (size_t)vi * 16) : make_uint4(0, 0, 0, 0);
  }
  unsigned long long best = 0;
  bool nan_seen = false;
  if (DT == DDTREE_BF16) {
    // pass 1: the chunk's largest value (bf16 widens to fp32 exactly with a
    // shift; fmaxf skips NaN, which the magnitude maxima below detect)
    float mx = -INFINITY;
    uint32_t mag_lo = 0, mag_hi = 0;
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      if (v * ARGMAX_THREADS + tid < nvec_full) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t w = u32_at(vec[v], q);
          mx = fmaxf(mx, fmaxf(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
          mag_lo = max(mag_lo, w & 0x7FFFu);
          mag_hi = max(mag_hi, w & 0x7FFF0000u);
        }
      }
    }
    for (int e = nvec_full * EPV + tid; e < len; e += ARGMAX_THREADS) {   // ragged tail
      const uint32_t bits = ((const uint16_t*)base)[e];
      mx = fmaxf(mx, bf16_bits_to_f32((uint16_t)bits));
      mag_lo = max(mag_lo, bits & 0x7FFFu);
    }
    nan_seen = mag_lo > 0x7F80u || mag_hi > 0x7F800000u;
    const float tmx = mx;
    mx = warp_max(mx);
    if ((tid & 31) == 0) redf[tid >> 5] = mx;
    __syncthreads();
    mx = redf[0];
#pragma unroll
    for (int i = 1; i < ARGMAX_THREADS / 32; ++i) mx = fmaxf(mx, redf[i]);
    // pass 2: the lowest chunk-local index holding the maximum (-0.0 == +0.0);
    // only threads that hold it scan
    uint32_t lowest = 0xFFFFFFFFu;
    if (tmx == mx) {
#pragma unroll
      for (int v = VPT - 1; v >= 0; --v) {           // later vectors first, so the lowest index wins
        const int vi = v * ARGMAX_THREADS + tid;
        if (vi < nvec_full) {
#pragma unroll
          for (int q = 3; q >= 0; --q) {
            const uint32_t w = u32_at(vec[v], q);
            if (__uint_as_float(w & 0xFFFF0000u) == mx) lowest = (uint32_t)(vi * EPV + 2 * q + 1);
            if (__uint_as_float(w << 16) == mx) lowest = (uint32_t)(vi * EPV + 2 * q);
          }
        }
      }
      for (int e = nvec_full * EPV + tid; e < len; e += ARGMAX_THREADS)
        if (bf16_bits_to_f32(((const uint16_t*)base)[e]) == mx) lowest = min(lowest, (uint32_t)e);
    }
    lowest = __reduce_min_sync(0xffffffffu, lowest);
    if ((tid & 31) == 0) red32[tid >> 5] = lowest;
    __syncthreads();
    uint32_t lmin = red32[0];
#pragma unroll
    for (int i = 1; i < ARGMAX_THREADS / 32; ++i) lmin = min(lmin, red32[i]);
    const uint32_t gid = (uint32_t)(c0 + lmin);
    best = ((unsigned long long)key32_of_f32(mx) << TOPK_ID_BITS) | (TOPK_ID_MASK - gid);
  } else {
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int vi = v * ARGMAX_THREADS + tid;
      if (vi < nvec_full) {
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
          const float f = __uint_as_float(u32_at(vec[v], j));
          nan_seen |= (f != f);
          const uint32_t gid = (uint32_t)(c0 + (long long)vi * EPV + j);
          const unsigned long long k = ((unsigned long long)key32_of_f32(f) << TOPK_ID_BITS) | (TOPK_ID_MASK - gid);
          best = k > best ? k : best;
        }
      }
    }
    for (int e = nvec_full * EPV + tid; e < len; e += ARGMAX_THREADS) {
      const float f = ((const float*)base)[e];
      nan_seen |= (f != f);
      const uint32_t gid = (uint32_t)(c0 + e);
      const unsigned long long k = ((unsigned long long)key32_of_f32(f) << TOPK_ID_BITS) | (TOPK_ID_MASK - gid);
      best = k > best ? k : best;
    }
    best = warp_max_u64(best);
  }
  if (__any_sync(0xffffffffu, nan_seen) && (tid & 31) == 0) flag_status(DDTREE_STATUS_NONFINITE);
  if ((tid & 31) == 0) red[tid >> 5] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long b = red[0];
    for (int i = 1; i < ARGMAX_THREADS / 32; ++i) b = red[i] > b ? red[i] : b;
    atomicMax(&ws.best[row], b);
    __threadfence();
    const unsigned t = atomicAdd(&ws.ticket[row], 1u);
    if (t == (unsigned)(cpr - 1)) {
      __threadfence();
      const unsigned long long fin = atomicExch(&ws.best[row], 0ull);   // read and reset
      ws.argmax[row] = (int32_t)(TOPK_ID_MASK - (uint32_t)(fin & TOPK_ID_MASK));
      ws.ticket[row] = 0;
    }
  }
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

__global__ void __launch_bounds__(WALK_THREADS) walk_compact_kernel(WalkArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int* nxt = (int*)smem_raw;          // [n]
  int* targ = nxt + a.n;              // [n]
  __shared__ int s_path[33];
  __shared__ int s_k;
  __shared__ int s_ok;
  const int r = blockIdx.x;
  const int lk = blockIdx.y;          // layer * 2 + (0: K, 1: V)
  const int tid = threadIdx.x;
  const int nn = a.n_nodes[r];
  const int P = a.prefix_len[r];
  const size_t ro = (size_t)r * a.n;
  for (int i = tid; i < nn; i += WALK_THREADS) {
    nxt[i] = -1;
    targ[i] = a.argmax_ws[ro + i];
  }
  __syncthreads();
  for (int j = 1 + tid; j < nn; j += WALK_THREADS) {
    const int p = a.parent[ro + j];
    if (a.node_token[ro + j] == targ[p]) nxt[p] = j;
  }
  __syncthreads();
  if (tid == 0) {
    int cur = 0, k = 0;
    s_path[0] = 0;
    while (k < a.L && nxt[cur] >= 0) {
      cur = nxt[cur];
      s_path[++k] = cur;
    }
    s_k = k;
    const long long cap = a.paged ? (long long)a.max_blocks * DDTREE_PAGE : (long long)a.s_max;
    s_ok = (P >= 0 && (long long)P + nn <= cap) ? 1 : 0;
  }
  __syncthreads();
  if (a.paged && a.k_cache != nullptr && s_ok) {   // blocks holding slots [0, P + nn) must be pool blocks
    const int nb = (P + nn + DDTREE_PAGE - 1) / DDTREE_PAGE;
    int bad = 0;
    for (int b = tid; b < nb; b += WALK_THREADS) {
      const int blk = a.block_table[(size_t)r * a.max_blocks + b];
      bad |= (blk < 0 || blk >= a.num_blocks);
    }
    bad = __syncthreads_or(bad);
    if (tid == 0 && bad) s_ok = 0;
    __syncthreads();
  }
  const int k = s_k;
  if (lk == 0) {
    for (int i = tid; i <= a.L; i += WALK_THREADS) {
      const bool on = i <= k;
      if (a.path) a.path[(size_t)r * (a.L + 1) + i] = on ? s_path[i] : -1;
      if (a.src_slot) a.src_slot[(size_t)r * (a.L + 1) + i] = on ? P + s_path[i] : -1;
      if (a.dst_slot) a.dst_slot[(size_t)r * (a.L + 1) + i] = on ? P + i : -1;
    }
    if (a.target_argmax)
      for (int i = tid; i < a.n; i += WALK_THREADS) a.target_argmax[ro + i] = i < nn ? targ[i] : -1;
    if (tid == 0) {
      if (a.accept_len) a.accept_len[r] = k + 1;
      if (a.next_bonus) a.next_bonus[r] = targ[s_path[k]];
      a.new_prefix_len[r] = P + k + 1;
      if (!s_ok && a.k_cache) flag_status(DDTREE_STATUS_CAPACITY);
    }
  }
  if (a.k_cache == nullptr || !s_ok || k == 0) return;

  // ---- compaction of this (layer, K/V) ----
  const int layer = lk >> 1;
  unsigned char* cache = (lk & 1) ? a.v_cache : a.k_cache;
  const int vec_per_row = a.row_bytes / 16;
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
  // rows j = 1..k move (row 0 is the root, already in place)
  const int total = k * vec_per_row;
  const int per_batch = WALK_THREADS * WALK_VPT;
  for (int b0 = 0; b0 < total; b0 += per_batch) {
    uint4 buf[WALK_VPT];
#pragma unroll
    for (int t = 0; t < WALK_VPT; ++t) {
      const int e = b0 + t * WALK_THREADS + tid;
      if (e < total) {
        const int j = 1 + e / vec_per_row, c = e % vec_per_row;
        buf[t] = *((const uint4*)row_ptr(P + s_path[j]) + c);
      }
    }
    __syncthreads();   // every source of this batch is read before any write
#pragma unroll
    for (int t = 0; t < WALK_VPT; ++t) {
      const int e = b0 + t * WALK_THREADS + tid;
      if (e < total) {
        const int j = 1 + e / vec_per_row, c = e % vec_per_row;
        if (s_path[j] != j) *((uint4*)row_ptr(P + j) + c) = buf[t];
      }
    }
    __syncthreads();
  }
}

}  // namespace ddt
