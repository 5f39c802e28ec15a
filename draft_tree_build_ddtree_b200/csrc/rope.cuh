// Verify-layer neighbour: the tree nodes' rotary positions and their K/V in
// the cache tail.
//
// "DDTree Deep Dive" §3 (tree_compile: every node gets the position id
// P + depth, so siblings share a position) and §5 (tree K/V sit in the
// cache tail, node i at slot P + i).  For each live node of each request and
// layer: Q (optional) and K are turned by the rotary position embedding at
// position P + depth (Su et al., "RoFormer", §3.4, half-split pairing: for
// i < D/2 the pair (x_i, x_{i+D/2}) turns by pos * theta^(-2i/D)), K and V
// are written into cache slot P + i, contiguous or paged.
//
// One CTA per (layer, request, node).  The node's D/2 angles are computed
// once in fp64 (pow, sincos) into shared memory as fp32 (cos, sin); every
// head row of Q, K and V of the node then moves as 16-byte vectors: one
// item rotates one vector of the first half with the matching vector of the
// second half.  HBM-bound: the inputs are read once, the outputs written
// once.
#pragma once

#include "common.cuh"

namespace ddt {

constexpr int ROPE_THREADS = 128;

struct RopeArgs {
  const unsigned char* q_in;    // [layers][n_req][n][Hq][D] or null
  unsigned char* q_out;         // same layout (may alias q_in)
  const unsigned char* k_in;    // [layers][n_req][n][Hkv][D]
  const unsigned char* v_in;
  const int32_t* depth;         // [n_req][n]
  const int32_t* n_nodes;       // [n_req]
  const int32_t* prefix_len;    // [n_req]
  const int32_t* block_table;   // paged: [n_req][max_blocks]
  unsigned char* k_cache;
  unsigned char* v_cache;
  int layers, n_req, n, Hq, Hkv, D;
  int paged, s_max, num_blocks, max_blocks;
  double theta;                 // <= 0: no rotation
};

template <typename T>
__global__ void __launch_bounds__(ROPE_THREADS) tree_rope_kernel(RopeArgs a) {
  constexpr int EPV = 16 / (int)sizeof(T);
  extern __shared__ float2 cs[];                        // [D/2] (cos, sin)
  int u = blockIdx.x;
  const int node = u % a.n; u /= a.n;
  const int r = u % a.n_req;
  const int layer = u / a.n_req;
  const int nn = a.n_nodes[r];
  if (node >= nn) return;
  const int P = a.prefix_len[r];
  const long long cap = a.paged ? (long long)a.max_blocks * DDTREE_PAGE : (long long)a.s_max;
  const int slot = P + node;
  size_t crow;                                          // cache row of the slot
  if (P < 0 || (long long)P + nn > cap) {
    if (threadIdx.x == 0 && node == 0 && layer == 0) flag_status(DDTREE_STATUS_CAPACITY);
    return;
  }
  if (a.paged) {
    const int blk = a.block_table[(size_t)r * a.max_blocks + slot / DDTREE_PAGE];
    if (blk < 0 || blk >= a.num_blocks) {
      if (threadIdx.x == 0) flag_status(DDTREE_STATUS_CAPACITY);
      return;
    }
    crow = ((size_t)layer * a.num_blocks + blk) * DDTREE_PAGE + (slot % DDTREE_PAGE);
  } else {
    crow = ((size_t)layer * a.n_req + r) * a.s_max + slot;
  }
  const int half = a.D / 2;
  const bool rotate = a.theta > 0.0;
  if (rotate) {
    const double pos = (double)(P + a.depth[(size_t)r * a.n + node]);
    for (int i = threadIdx.x; i < half; i += ROPE_THREADS) {
      const double inv = pow(a.theta, -(2.0 * i) / (double)a.D);
      double sn, cn;
      sincos(pos * inv, &sn, &cn);
      cs[i] = make_float2((float)cn, (float)sn);
    }
    __syncthreads();
  }
  const size_t row_bytes_q = (size_t)a.Hq * a.D * sizeof(T);
  const size_t row_bytes_kv = (size_t)a.Hkv * a.D * sizeof(T);
  const size_t nrow = ((size_t)layer * a.n_req + r) * a.n + node;   // input row of (layer, request, node)
  const int vph = half / EPV;                           // vectors per half row
  const int qheads = a.q_in != nullptr ? a.Hq : 0;
  const int rot_items = (qheads + a.Hkv) * vph;         // Q rows then K rows, one pair of vectors each
  const int copy_items = a.Hkv * 2 * vph;               // V rows, whole vectors
  for (int it = threadIdx.x; it < rot_items + copy_items; it += ROPE_THREADS) {
    if (it < rot_items) {
      const int h = it / vph, c = it - h * vph;
      const bool is_q = h < qheads;
      const int head = is_q ? h : h - qheads;
      const unsigned char* src = is_q ? a.q_in + nrow * row_bytes_q : a.k_in + nrow * row_bytes_kv;
      unsigned char* dst = is_q ? a.q_out + nrow * row_bytes_q : a.k_cache + crow * row_bytes_kv;
      const size_t o0 = ((size_t)head * a.D + (size_t)c * EPV) * sizeof(T);
      const size_t o1 = o0 + (size_t)half * sizeof(T);
      uint4 va = *reinterpret_cast<const uint4*>(src + o0);
      uint4 vb = *reinterpret_cast<const uint4*>(src + o1);
      if (rotate) {
        T* xa = reinterpret_cast<T*>(&va);
        T* xb = reinterpret_cast<T*>(&vb);
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
          const float2 t = cs[c * EPV + e];
          const float fa = (float)xa[e], fb = (float)xb[e];
          xa[e] = (T)(fa * t.x - fb * t.y);
          xb[e] = (T)(fb * t.x + fa * t.y);
        }
      }
      *reinterpret_cast<uint4*>(dst + o0) = va;
      *reinterpret_cast<uint4*>(dst + o1) = vb;
    } else {
      const int k = it - rot_items;                     // vector k of the node's V row
      const size_t o = (size_t)k * 16;
      *reinterpret_cast<uint4*>(a.v_cache + crow * row_bytes_kv + o) =
          *reinterpret_cast<const uint4*>(a.v_in + nrow * row_bytes_kv + o);
    }
  }
}

}  // namespace ddt
