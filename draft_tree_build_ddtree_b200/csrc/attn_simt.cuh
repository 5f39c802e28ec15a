// Stage 3 (CUDA-core path): ancestor-only tree attention, one warp per
// (layer, request, node, query head).
//
// "DDTree Deep Dive" §4: node i attends to the committed prefix, the root,
// its ancestors and itself, never to siblings.  Keys are the prefix slots
// 0..P-1 and the tree slots P+j for every j set in the node's ancestor
// bitmask.
//
// This path serves fp32 inputs and head_dim 64, and is the reference the
// tensor-core kernel is debugged against.  Scores use lane-per-key dot
// products (32 keys per step, q broadcast from shared memory), an online
// softmax in fp32, and the PV product with each lane owning D/32
// consecutive output dimensions.
#pragma once

#include "common.cuh"

namespace ddt {

constexpr int ATTN_SIMT_WARPS = 4;

struct AttnGeom {
  int layers, n_req, n, Hq, Hkv, D, W;
  float scale;
  int paged, s_max, num_blocks, max_blocks;
};

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Row index (in units of Hkv*D elements) of logical slot `slot` of request r.
__device__ __forceinline__ size_t kv_row(const AttnGeom& g, const int32_t* block_table, int layer, int r,
                                         int slot) {
  if (g.paged) {
    const int blk = block_table[(size_t)r * g.max_blocks + slot / DDTREE_PAGE];
    return ((size_t)layer * g.num_blocks + blk) * DDTREE_PAGE + (slot % DDTREE_PAGE);
  }
  return ((size_t)layer * g.n_req + r) * g.s_max + slot;
}

template <typename T, int D>
__global__ void __launch_bounds__(ATTN_SIMT_WARPS * 32)
tree_attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                      const int32_t* __restrict__ block_table, const int32_t* __restrict__ prefix_len,
                      const uint32_t* __restrict__ anc, const int32_t* __restrict__ n_nodes, AttnGeom g,
                      T* __restrict__ out, float* __restrict__ out_lse) {
  constexpr int DPL = D / 32;   // output dims per lane
  __shared__ float qs[ATTN_SIMT_WARPS][D];
  __shared__ int vis[33];
  __shared__ int s_nvis;
  const int hgroups = (g.Hq + ATTN_SIMT_WARPS - 1) / ATTN_SIMT_WARPS;
  int b = blockIdx.x;
  const int hg = b % hgroups; b /= hgroups;
  const int i = b % g.n; b /= g.n;
  const int r = b % g.n_req; b /= g.n_req;
  const int layer = b;
  const int nn = n_nodes[r];
  if (i >= nn) return;
  const int P = prefix_len[r];
  const long long cap = g.paged ? (long long)g.max_blocks * DDTREE_PAGE : (long long)g.s_max;
  if (P < 0 || (long long)P + nn > cap) {
    if (threadIdx.x == 0 && i == 0 && hg == 0) flag_status(DDTREE_STATUS_CAPACITY);
    return;
  }
  if (g.paged) {   // every block the request reads must be a pool block
    const int nb = (P + nn + DDTREE_PAGE - 1) / DDTREE_PAGE;
    int bad = 0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
      const int blk = block_table[(size_t)r * g.max_blocks + b];
      bad |= (blk < 0 || blk >= g.num_blocks);
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0 && i == 0 && hg == 0) flag_status(DDTREE_STATUS_CAPACITY);
      return;
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int c = 0;
    const uint32_t* arow = anc + ((size_t)r * g.n + i) * g.W;
    for (int w = 0; w < g.W; ++w) {
      uint32_t bits = arow[w];
      while (bits && c < 33) {
        const int t = __ffs(bits) - 1;
        bits &= bits - 1;
        vis[c++] = 32 * w + t;
      }
    }
    s_nvis = c;
  }
  const int h = hg * ATTN_SIMT_WARPS + warp;
  const bool active = h < g.Hq;
  const size_t qrow = ((((size_t)layer * g.n_req + r) * g.n + i) * g.Hq + (active ? h : 0)) * D;
  for (int d = lane; d < D; d += 32) qs[warp][d] = active ? to_f(q[qrow + d]) : 0.f;
  __syncthreads();
  if (!active) return;
  const int kvh = h / (g.Hq / g.Hkv);
  const int nvis = s_nvis;
  const int T_all = P + nvis;
  const size_t rstride = (size_t)g.Hkv * D;

  float m = -INFINITY, l = 0.f;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;

  for (int t0 = 0; t0 < T_all; t0 += 32) {
    const int t = t0 + lane;
    const bool valid = t < T_all;
    const int slot = valid ? (t < P ? t : P + vis[t - P]) : 0;
    float s = -INFINITY;
    if (valid) {
      const T* kr = kc + kv_row(g, block_table, layer, r, slot) * rstride + (size_t)kvh * D;
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) dot = fmaf(qs[warp][d], to_f(kr[d]), dot);
      s = dot * g.scale;
    }
    const float mb = warp_max(s);
    const float mn = fmaxf(m, mb);
    const float p = valid ? expf(s - mn) : 0.f;
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    l = l * corr + warp_sum(p);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] *= corr;
    m = mn;
    const int cnt = min(32, T_all - t0);
    for (int u = 0; u < cnt; ++u) {
      const float pu = __shfl_sync(0xffffffffu, p, u);
      const int su = __shfl_sync(0xffffffffu, slot, u);
      const T* vr = vc + kv_row(g, block_table, layer, r, su) * rstride + (size_t)kvh * D + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pu, to_f(vr[e]), acc[e]);
    }
  }
  const float inv = 1.f / l;
  T* orow = out + qrow + lane * DPL;
#pragma unroll
  for (int e = 0; e < DPL; ++e) orow[e] = from_f<T>(acc[e] * inv);
  if (out_lse && lane == 0)
    out_lse[(((size_t)layer * g.n_req + r) * g.n + i) * g.Hq + h] = m + logf(l);
}

}  // namespace ddt
