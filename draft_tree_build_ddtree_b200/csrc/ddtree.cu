// libddtree.so: the C ABI of include/ddtree.h.
//
// One translation unit: the kernels of every stage are included here so the
// device status word is a single symbol without relocatable device code.
// Host code validates every argument before launching anything; kernels
// never trap, assert or wait on another CTA.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "ddtree.h"
#include "common.cuh"
#include "topk.cuh"
#include "build.cuh"
#include "accept.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "attn_tc2.cuh"
#include "rope.cuh"
#include "lmhead.cuh"

using namespace ddt;

namespace {

constexpr int MAX_L = 32;
constexpr int MAX_K = 1024;
constexpr int MAX_B = 1024;
constexpr int MAX_REQ = 4096;
constexpr int MAX_V = 1 << TOPK_ID_BITS;

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int max_smem_optin() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return n > 0 ? n : 227 * 1024;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int esize_of(int dtype) { return dtype == DDTREE_BF16 ? 2 : 4; }

bool dtype_ok(int dtype) { return dtype == DDTREE_BF16 || dtype == DDTREE_F32; }

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DDTREE_OK : cuda_fail(e, "kernel launch");
}

// Opt a kernel in to `bytes` of dynamic shared memory when its static plus
// dynamic shared memory exceeds the default 48 KB; the attribute is raised
// once per kernel and size (cached per device-independent function pointer).
struct SmemOptIn {
  const void* fn;
  size_t bytes;
};
SmemOptIn g_smem_optin[64];
int g_smem_optin_n = 0;

template <typename F>
int set_smem(F* kernel, size_t bytes) {
  const void* fn = (const void*)kernel;
  int slot = -1;
  for (int i = 0; i < g_smem_optin_n; ++i)
    if (g_smem_optin[i].fn == fn) slot = i;
  if (slot >= 0 && g_smem_optin[slot].bytes >= bytes) return DDTREE_OK;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return DDTREE_ERR_CUDA;
  if (bytes + attr.sharedSizeBytes > (size_t)max_smem_optin()) return DDTREE_ERR_UNSUPPORTED;
  if (bytes + attr.sharedSizeBytes > 48 * 1024) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
      return DDTREE_ERR_CUDA;
  }
  if (slot < 0 && g_smem_optin_n < 64) slot = g_smem_optin_n++;
  if (slot >= 0) g_smem_optin[slot] = SmemOptIn{fn, bytes};
  return DDTREE_OK;
}

// ------------------------------------------------------------------ topk
// The exp(z) table of every bf16 value is built once per device, on the
// first bf16 top-K call, which then synchronizes its stream once (inside a
// stream capture the build is captured instead: it is idempotent).
constexpr int EXP_TABLE_MAX_DEVICES = 64;
bool g_exp_table_ready[EXP_TABLE_MAX_DEVICES];

int ensure_exp_table(cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= EXP_TABLE_MAX_DEVICES) return DDTREE_ERR_CUDA;
  if (g_exp_table_ready[dev]) return DDTREE_OK;
  exp_bf16_table_kernel<<<65536 / 256, 256, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return DDTREE_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return DDTREE_ERR_CUDA;
  if (cs == cudaStreamCaptureStatusNone) {
    if (cudaStreamSynchronize(s) != cudaSuccess) return DDTREE_ERR_CUDA;
    g_exp_table_ready[dev] = true;
  }
  return DDTREE_OK;
}

int topk_check(const void* logits, int dtype, int rows, int V, long long row_stride, int K,
               const void* ids, const void* lp) {
  if (!logits || !ids || !lp) return DDTREE_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return DDTREE_ERR_INVALID_ARG;
  if (rows < 1 || V < 1 || V > MAX_V || K < 1 || K > MAX_K || K > V) return DDTREE_ERR_INVALID_ARG;
  if (row_stride < V || (row_stride * esize_of(dtype)) % 16 != 0) return DDTREE_ERR_INVALID_ARG;
  if (!aligned16(logits)) return DDTREE_ERR_INVALID_ARG;
  return DDTREE_OK;
}

size_t topk_ws(int rows, int V, int K, int dtype) {
  TopkPlan p = topk_plan(rows, V, K, esize_of(dtype), num_sms());
  return topk_ws_bytes(rows, p);
}

int topk_launch(const void* logits, int dtype, int rows, int V, long long row_stride, int K,
                int32_t* ids, float* lp, float* lse, void* ws, size_t ws_bytes, cudaStream_t s) {
  int st = topk_check(logits, dtype, rows, V, row_stride, K, ids, lp);
  if (st) return st;
  TopkPlan p = topk_plan(rows, V, K, esize_of(dtype), num_sms());
  if (p.cpr == 0 || p.cand > TOPK_MAX_CAND) return DDTREE_ERR_UNSUPPORTED;
  if (!ws || !aligned16(ws) || ws_bytes < topk_ws_bytes(rows, p)) return DDTREE_ERR_INVALID_ARG;
  TopkWs w = topk_ws_carve(ws, rows, p);
  const size_t smem = topk_smem_bytes(p, K);
  const long long grid = (long long)rows * p.cpr;
  if (grid > 0x7fffffffLL) return DDTREE_ERR_UNSUPPORTED;
  if (dtype == DDTREE_BF16) {
    if ((st = ensure_exp_table(s))) return st;
    switch (p.vpt) {
#define DDT_TOPK_CASE(VP)                                                                                   \
  case VP:                                                                                                  \
    if ((st = set_smem(topk_kernel<DDTREE_BF16, VP>, smem))) return st;                                     \
    topk_kernel<DDTREE_BF16, VP><<<(unsigned)grid, TOPK_THREADS, smem, s>>>(logits, rows, V, row_stride, K, \
                                                                            p, w, ids, lp, lse);            \
    break;
      DDT_TOPK_CASE(1) DDT_TOPK_CASE(2) DDT_TOPK_CASE(3) DDT_TOPK_CASE(4) DDT_TOPK_CASE(5) DDT_TOPK_CASE(6)
#undef DDT_TOPK_CASE
      default: return DDTREE_ERR_UNSUPPORTED;
    }
  } else {
    switch (p.vpt) {
#define DDT_TOPK_CASE(VP)                                                                                  \
  case VP:                                                                                                 \
    if ((st = set_smem(topk_kernel<DDTREE_F32, VP>, smem))) return st;                                     \
    topk_kernel<DDTREE_F32, VP><<<(unsigned)grid, TOPK_THREADS, smem, s>>>(logits, rows, V, row_stride, K, \
                                                                           p, w, ids, lp, lse);            \
    break;
      DDT_TOPK_CASE(1) DDT_TOPK_CASE(2) DDT_TOPK_CASE(3) DDT_TOPK_CASE(4) DDT_TOPK_CASE(5) DDT_TOPK_CASE(6)
#undef DDT_TOPK_CASE
      default: return DDTREE_ERR_UNSUPPORTED;
    }
  }
  return launch_status();
}

// ------------------------------------------------------------------ build
int build_launch(const int32_t* ids, const float* lp, const int32_t* root_token, int n_req, int L, int K,
                 int B, int32_t* node_token, int32_t* parent, int32_t* depth, int32_t* node_rank,
                 float* score, uint32_t* anc, int32_t* n_nodes, cudaStream_t s, int flags = 0,
                 const float* gain_floor = nullptr, int32_t* build_path = nullptr) {
  if (!ids || !lp || !root_token || !parent || !anc || !n_nodes) return DDTREE_ERR_INVALID_ARG;
  if (n_req < 1 || n_req > MAX_REQ || L < 1 || L > MAX_L || K < 1 || K > MAX_K || B < 0 || B > MAX_B)
    return DDTREE_ERR_INVALID_ARG;
  if (flags & ~DDTREE_BUILD_FORCE_HEAP) return DDTREE_ERR_INVALID_ARG;
  const int kc = B < K ? B : K;
  // the threshold enumeration when its arrays fit beside the heap's
  const int nt = build_threads(B);
  auto kern = nt == BUILD_THREADS_LARGE ? build_kernel<BUILD_THREADS_LARGE> : build_kernel<BUILD_THREADS_SMALL>;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return DDTREE_ERR_CUDA;
  const size_t smem_enum = build_smem_bytes_enum(L, kc, B);
  const int use_enum =
      (!(flags & DDTREE_BUILD_FORCE_HEAP) && smem_enum + attr.sharedSizeBytes <= (size_t)max_smem_optin()) ? 1 : 0;
  const size_t smem = use_enum ? smem_enum : build_smem_bytes(L, kc, B);
  int st = set_smem(kern, smem);
  if (st) return st;
  kern<<<n_req, nt, smem, s>>>(ids, lp, root_token, L, K, B, kc, tie_code(kc, L), use_enum,
                                                   gain_floor, node_token, parent, depth, node_rank, score, anc,
                                                   n_nodes, build_path);
  return launch_status();
}

// ------------------------------------------------------------------ attention
int kv_check(const ddtree_kv_desc* kv) {
  if (!kv) return DDTREE_ERR_INVALID_ARG;
  if (kv->layers < 1 || kv->n_req < 1 || kv->n_req > MAX_REQ || kv->Hq < 1 || kv->Hkv < 1 ||
      kv->Hq % kv->Hkv != 0)
    return DDTREE_ERR_INVALID_ARG;
  if (kv->D != 64 && kv->D != 128) return DDTREE_ERR_UNSUPPORTED;
  if (kv->paged) {
    if (kv->num_blocks < 1 || kv->max_blocks < 1) return DDTREE_ERR_INVALID_ARG;
  } else if (kv->s_max < 1) {
    return DDTREE_ERR_INVALID_ARG;
  }
  return DDTREE_OK;
}

AttnGeom geom_of(const ddtree_kv_desc* kv, int B) {
  AttnGeom g;
  g.layers = kv->layers;
  g.n_req = kv->n_req;
  g.n = B + 1;
  g.Hq = kv->Hq;
  g.Hkv = kv->Hkv;
  g.D = kv->D;
  g.W = (B + 1 + 31) / 32;
  g.scale = kv->scale > 0.f ? kv->scale : 1.0f / sqrtf((float)kv->D);
  g.paged = kv->paged;
  g.s_max = kv->s_max;
  g.num_blocks = kv->num_blocks;
  g.max_blocks = kv->max_blocks;
  return g;
}

// Diagnostics of the attention pipeline's timeout path (ddtree_debug_attn_timeout).
unsigned long long g_attn_wait_ns = 0;   // 0: the default limit
int g_attn_stop_tile = -1;

bool use_tc_attn(int dtype, const ddtree_kv_desc* kv) {
  return dtype == DDTREE_BF16 && (kv->D == 128 || kv->D == 64) && tc_attn_supported(kv->Hq / kv->Hkv);
}

size_t attn_ws(const ddtree_kv_desc* kv, int B, int dtype) {
  if (!use_tc_attn(dtype, kv)) return 0;
  return attn_tc_ws_bytes(geom_of(kv, B), num_sms());
}

int attn_launch(const void* q, const void* k_cache, const void* v_cache, int dtype, const ddtree_kv_desc* kv,
                const int32_t* block_table, const int32_t* prefix_len, const uint32_t* anc,
                const int32_t* n_nodes, int B, void* out, float* out_lse, void* ws, size_t ws_bytes,
                cudaStream_t s, int early = 0) {
  int st = kv_check(kv);
  if (st) return st;
  if (!dtype_ok(dtype) || B < 0 || B > MAX_B) return DDTREE_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !prefix_len || !anc || !n_nodes || !out) return DDTREE_ERR_INVALID_ARG;
  if (kv->paged && !block_table) return DDTREE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return DDTREE_ERR_INVALID_ARG;
  AttnGeom g = geom_of(kv, B);
  if (use_tc_attn(dtype, kv)) {
    const size_t need = attn_tc_ws_bytes(g, num_sms());
    if (need && (!ws || !aligned16(ws) || ws_bytes < need)) return DDTREE_ERR_INVALID_ARG;
    return attn_tc_launch(q, k_cache, v_cache, block_table, prefix_len, anc, n_nodes, g, out, out_lse, ws,
                          num_sms(), s, g_attn_wait_ns, g_attn_stop_tile, early);
  }
  const long long grid =
      (long long)g.layers * g.n_req * g.n * ((g.Hq + ATTN_SIMT_WARPS - 1) / ATTN_SIMT_WARPS);
  if (grid > 0x7fffffffLL) return DDTREE_ERR_UNSUPPORTED;
  const dim3 blk(ATTN_SIMT_WARPS * 32);
  if (dtype == DDTREE_BF16) {
    typedef __nv_bfloat16 T;
    if (g.D == 64)
      tree_attn_simt_kernel<T, 64><<<(unsigned)grid, blk, 0, s>>>((const T*)q, (const T*)k_cache,
                                                                  (const T*)v_cache, block_table, prefix_len,
                                                                  anc, n_nodes, g, (T*)out, out_lse);
    else
      tree_attn_simt_kernel<T, 128><<<(unsigned)grid, blk, 0, s>>>((const T*)q, (const T*)k_cache,
                                                                   (const T*)v_cache, block_table, prefix_len,
                                                                   anc, n_nodes, g, (T*)out, out_lse);
  } else {
    typedef float T;
    if (g.D == 64)
      tree_attn_simt_kernel<T, 64><<<(unsigned)grid, blk, 0, s>>>((const T*)q, (const T*)k_cache,
                                                                  (const T*)v_cache, block_table, prefix_len,
                                                                  anc, n_nodes, g, (T*)out, out_lse);
    else
      tree_attn_simt_kernel<T, 128><<<(unsigned)grid, blk, 0, s>>>((const T*)q, (const T*)k_cache,
                                                                   (const T*)v_cache, block_table, prefix_len,
                                                                   anc, n_nodes, g, (T*)out, out_lse);
  }
  return launch_status();
}

// ------------------------------------------------------------------ tree K/V write with rotary positions
int rope_launch(const void* q_in, void* q_out, const void* k_in, const void* v_in, int dtype, const int32_t* depth,
                const int32_t* n_nodes, const int32_t* prefix_len, const ddtree_kv_desc* kv,
                const int32_t* block_table, int B, double theta, void* k_cache, void* v_cache, cudaStream_t s) {
  int st = kv_check(kv);
  if (st) return st;
  if (!dtype_ok(dtype) || B < 0 || B > MAX_B) return DDTREE_ERR_INVALID_ARG;
  if (!k_in || !v_in || !depth || !n_nodes || !prefix_len || !k_cache || !v_cache) return DDTREE_ERR_INVALID_ARG;
  if ((q_in == nullptr) != (q_out == nullptr)) return DDTREE_ERR_INVALID_ARG;
  if (kv->paged && !block_table) return DDTREE_ERR_INVALID_ARG;
  if (theta != theta) return DDTREE_ERR_INVALID_ARG;
  for (const void* p : {(const void*)q_in, (const void*)q_out, k_in, v_in, (const void*)k_cache, (const void*)v_cache})
    if (p && !aligned16(p)) return DDTREE_ERR_INVALID_ARG;
  RopeArgs a;
  a.q_in = (const unsigned char*)q_in;
  a.q_out = (unsigned char*)q_out;
  a.k_in = (const unsigned char*)k_in;
  a.v_in = (const unsigned char*)v_in;
  a.depth = depth;
  a.n_nodes = n_nodes;
  a.prefix_len = prefix_len;
  a.block_table = block_table;
  a.k_cache = (unsigned char*)k_cache;
  a.v_cache = (unsigned char*)v_cache;
  a.layers = kv->layers;
  a.n_req = kv->n_req;
  a.n = B + 1;
  a.Hq = kv->Hq;
  a.Hkv = kv->Hkv;
  a.D = kv->D;
  a.paged = kv->paged;
  a.s_max = kv->s_max;
  a.num_blocks = kv->num_blocks;
  a.max_blocks = kv->max_blocks;
  a.theta = theta;
  const long long grid = (long long)a.layers * a.n_req * a.n;
  if (grid > 0x7fffffffLL) return DDTREE_ERR_UNSUPPORTED;
  const size_t smem = (size_t)(kv->D / 2) * sizeof(float2);
  if (dtype == DDTREE_BF16)
    tree_rope_kernel<__nv_bfloat16><<<(unsigned)grid, ROPE_THREADS, smem, s>>>(a);
  else
    tree_rope_kernel<float><<<(unsigned)grid, ROPE_THREADS, smem, s>>>(a);
  return launch_status();
}

// ------------------------------------------------------------------ accept
struct AcceptPlan {
  int cpr, chunk;
};

// Chunks per row: about one wave of resident CTAs over all rows.
AcceptPlan accept_plan(int rows, int V) {
  const int resident = num_sms() * ARGMAX_CTAS_PER_SM;
  int cpr = resident / (rows > 0 ? rows : 1);
  const int cpr_small = ceil_div(V, 4096);
  if (cpr > cpr_small) cpr = cpr_small;
  if (cpr < 1) cpr = 1;
  AcceptPlan p;
  p.chunk = ceil_div(ceil_div(V, cpr), 8) * 8;
  p.cpr = ceil_div(V, p.chunk);
  return p;
}

size_t accept_ws(int n_req, int B) { return argmax_ws_bytes(n_req * (B + 1), n_req); }

int accept_launch(const void* target_logits, int dtype, int V, long long row_stride, const int32_t* node_token,
                  const int32_t* parent, const int32_t* n_nodes, int n_req, int L, int B,
                  const int32_t* prefix_len, int32_t* new_prefix_len, void* k_cache, void* v_cache,
                  const ddtree_kv_desc* kv, const int32_t* block_table, int32_t* target_argmax, int32_t* path,
                  int32_t* accept_len, int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot, void* ws,
                  size_t ws_bytes, cudaStream_t s, const ddtree_sampling* sampling = nullptr) {
  if (!target_logits || !node_token || !parent || !n_nodes || !prefix_len || !new_prefix_len)
    return DDTREE_ERR_INVALID_ARG;
  const bool sample = sampling != nullptr && sampling->temperature > 0.0;
  if (sampling != nullptr && !(sampling->temperature <= 0.0 || sampling->temperature < INFINITY))
    return DDTREE_ERR_INVALID_ARG;   // NaN or +inf temperature
  SampleArgs sa;
  sa.inv_t = sample ? 1.0 / sampling->temperature : 0.0;
  sa.seed = sample ? sampling->seed : 0ull;
  sa.offset = sample ? sampling->offset : 0ull;
  if (new_prefix_len == prefix_len) return DDTREE_ERR_INVALID_ARG;
  if (!dtype_ok(dtype) || V < 1 || V > MAX_V || n_req < 1 || n_req > MAX_REQ || L < 1 || L > MAX_L || B < 0 ||
      B > MAX_B)
    return DDTREE_ERR_INVALID_ARG;
  if (row_stride < V || (row_stride * esize_of(dtype)) % 16 != 0 || !aligned16(target_logits))
    return DDTREE_ERR_INVALID_ARG;
  const int n = B + 1;
  const int rows = n_req * n;
  if (!ws || !aligned16(ws) || ws_bytes < argmax_ws_bytes(rows, n_req)) return DDTREE_ERR_INVALID_ARG;
  int row_bytes = 0;
  if (k_cache) {
    int st = kv_check(kv);
    if (st) return st;
    if (!v_cache || kv->n_req != n_req || (kv->paged && !block_table)) return DDTREE_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return DDTREE_ERR_INVALID_ARG;
    row_bytes = kv->Hkv * kv->D * esize_of(dtype);
    if (row_bytes % 16 != 0) return DDTREE_ERR_UNSUPPORTED;
  }
  AcceptPlan p = accept_plan(rows, V);
  ArgmaxWs w = argmax_ws_carve(ws, rows);
  const long long grid = (long long)rows * p.cpr;
  if (grid > 0x7fffffffLL) return DDTREE_ERR_UNSUPPORTED;
  WalkArgs a;
  a.node_token = node_token;
  a.parent = parent;
  a.n_nodes = n_nodes;
  a.prefix_len = prefix_len;
  a.argmax_ws = w.argmax;
  a.n = n;
  a.L = L;
  a.new_prefix_len = new_prefix_len;
  a.target_argmax = target_argmax;
  a.path = path;
  a.accept_len = accept_len;
  a.next_bonus = next_bonus;
  a.src_slot = src_slot;
  a.dst_slot = dst_slot;
  a.k_cache = (unsigned char*)k_cache;
  a.v_cache = (unsigned char*)v_cache;
  a.block_table = block_table;
  a.layers = k_cache ? kv->layers : 1;
  a.n_req = n_req;
  a.paged = k_cache ? kv->paged : 0;
  a.s_max = k_cache ? kv->s_max : 0;
  a.num_blocks = k_cache ? kv->num_blocks : 0;
  a.max_blocks = k_cache ? kv->max_blocks : 0;
  a.row_bytes = row_bytes;
  // few layers: the CTA that publishes a request's last argmax walks and compacts it
  const int fuse = (!k_cache || kv->layers <= WALK_FUSE_MAX_LAYERS) ? 1 : 0;
#define DDT_ARGMAX(DT, SM)                                                                               \
  argmax_kernel<DT, SM><<<(unsigned)grid, ARGMAX_THREADS, 0, s>>>(target_logits, n, V, row_stride, n_nodes, \
                                                                  p.cpr, p.chunk, w, a, fuse, sa)
  if (dtype == DDTREE_BF16) {
    if (sample) DDT_ARGMAX(DDTREE_BF16, true); else DDT_ARGMAX(DDTREE_BF16, false);
  } else {
    if (sample) DDT_ARGMAX(DDTREE_F32, true); else DDT_ARGMAX(DDTREE_F32, false);
  }
#undef DDT_ARGMAX
  int st = launch_status();
  if (st || fuse) return st;
  const size_t smem = (size_t)n * 16;   // next, argmax, parent, token
  dim3 grid2(n_req, a.layers * 2);
  walk_compact_kernel<<<grid2, WALK_THREADS, smem, s>>>(a);
  return launch_status();
}

// ------------------------------------------------------------------ LM head + walk
int lmhead_check(const void* hidden, const void* weight, int rows, int V, int d, const void* out) {
  if (!hidden || !weight || !out) return DDTREE_ERR_INVALID_ARG;
  if (rows < 1 || rows > MAX_REQ * (MAX_B + 1) || V < 1 || V > MAX_V || d < 64 || d % 64 != 0 || d > 65536)
    return DDTREE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(weight)) return DDTREE_ERR_INVALID_ARG;
  return DDTREE_OK;
}

// The walk and compaction from given per-node target tokens (target_token
// [n_req][B+1]): one CTA per (request, layer, K/V).
int walk_launch(const int32_t* target_token, const int32_t* node_token, const int32_t* parent,
                const int32_t* n_nodes, int n_req, int L, int B, const int32_t* prefix_len, int32_t* new_prefix_len,
                void* k_cache, void* v_cache, const ddtree_kv_desc* kv, const int32_t* block_table, int dtype,
                int32_t* path, int32_t* accept_len, int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot,
                cudaStream_t s) {
  if (!target_token || !node_token || !parent || !n_nodes || !prefix_len || !new_prefix_len)
    return DDTREE_ERR_INVALID_ARG;
  if (new_prefix_len == prefix_len || !dtype_ok(dtype)) return DDTREE_ERR_INVALID_ARG;
  if (n_req < 1 || n_req > MAX_REQ || L < 1 || L > MAX_L || B < 0 || B > MAX_B) return DDTREE_ERR_INVALID_ARG;
  int row_bytes = 0;
  if (k_cache) {
    int st = kv_check(kv);
    if (st) return st;
    if (!v_cache || kv->n_req != n_req || (kv->paged && !block_table)) return DDTREE_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return DDTREE_ERR_INVALID_ARG;
    row_bytes = kv->Hkv * kv->D * esize_of(dtype);
    if (row_bytes % 16 != 0) return DDTREE_ERR_UNSUPPORTED;
  }
  WalkArgs a;
  a.node_token = node_token;
  a.parent = parent;
  a.n_nodes = n_nodes;
  a.prefix_len = prefix_len;
  a.argmax_ws = target_token;
  a.n = B + 1;
  a.L = L;
  a.new_prefix_len = new_prefix_len;
  a.target_argmax = nullptr;
  a.path = path;
  a.accept_len = accept_len;
  a.next_bonus = next_bonus;
  a.src_slot = src_slot;
  a.dst_slot = dst_slot;
  a.k_cache = (unsigned char*)k_cache;
  a.v_cache = (unsigned char*)v_cache;
  a.block_table = block_table;
  a.layers = k_cache ? kv->layers : 1;
  a.n_req = n_req;
  a.paged = k_cache ? kv->paged : 0;
  a.s_max = k_cache ? kv->s_max : 0;
  a.num_blocks = k_cache ? kv->num_blocks : 0;
  a.max_blocks = k_cache ? kv->max_blocks : 0;
  a.row_bytes = row_bytes;
  const size_t smem = (size_t)(B + 1) * 16;
  dim3 grid2(n_req, a.layers * 2);
  walk_compact_kernel<<<grid2, WALK_THREADS, smem, s>>>(a);
  return launch_status();
}

}  // namespace

// ======================================================================
// C ABI
// ======================================================================
extern "C" {

size_t ddtree_topk_workspace_bytes(int rows, int V, int K) {
  if (rows < 1 || V < 1 || K < 1) return 0;
  size_t a = topk_ws(rows, V, K, DDTREE_BF16), b = topk_ws(rows, V, K, DDTREE_F32);
  return a > b ? a : b;
}

int ddtree_topk(const void* logits, int dtype, int rows, int V, long long row_stride, int K, int32_t* ids,
                float* lp, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return topk_launch(logits, dtype, rows, V, row_stride, K, ids, lp, lse, ws, ws_bytes, stream);
}

int ddtree_build(const int32_t* ids, const float* lp, const int32_t* root_token, int n_req, int L, int K, int B,
                 int32_t* node_token, int32_t* parent, int32_t* depth, int32_t* node_rank, float* score,
                 uint32_t* anc, int32_t* n_nodes, cudaStream_t stream) {
  return build_launch(ids, lp, root_token, n_req, L, K, B, node_token, parent, depth, node_rank, score, anc,
                      n_nodes, stream);
}

int ddtree_build_ex(const int32_t* ids, const float* lp, const int32_t* root_token, int n_req, int L, int K, int B,
                    int32_t* node_token, int32_t* parent, int32_t* depth, int32_t* node_rank, float* score,
                    uint32_t* anc, int32_t* n_nodes, const float* gain_floor, int flags, int32_t* build_path,
                    cudaStream_t stream) {
  return build_launch(ids, lp, root_token, n_req, L, K, B, node_token, parent, depth, node_rank, score, anc,
                      n_nodes, stream, flags, gain_floor, build_path);
}

int ddtree_tree_kv_write(const void* q_in, void* q_out, const void* k_in, const void* v_in, int dtype,
                         const int32_t* depth, const int32_t* n_nodes, const int32_t* prefix_len,
                         const ddtree_kv_desc* kv, const int32_t* block_table, int B, double rope_theta,
                         void* k_cache, void* v_cache, cudaStream_t stream) {
  return rope_launch(q_in, q_out, k_in, v_in, dtype, depth, n_nodes, prefix_len, kv, block_table, B, rope_theta,
                     k_cache, v_cache, stream);
}

size_t ddtree_attn_workspace_bytes(const ddtree_kv_desc* kv, int B) {
  if (kv_check(kv) || B < 0 || B > MAX_B) return 0;
  return attn_ws(kv, B, DDTREE_BF16);
}

int ddtree_tree_attn(const void* q, const void* k_cache, const void* v_cache, int dtype, const ddtree_kv_desc* kv,
                     const int32_t* block_table, const int32_t* prefix_len, const uint32_t* anc,
                     const int32_t* n_nodes, int B, void* out, float* out_lse, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  return attn_launch(q, k_cache, v_cache, dtype, kv, block_table, prefix_len, anc, n_nodes, B, out, out_lse,
                     ws, ws_bytes, stream);
}

int ddtree_accept_ex(const void* target_logits, int dtype, int V, long long row_stride, const int32_t* node_token,
                     const int32_t* parent, const int32_t* n_nodes, int n_req, int L, int B,
                     const int32_t* prefix_len, int32_t* new_prefix_len, void* k_cache, void* v_cache,
                     const ddtree_kv_desc* kv, const int32_t* block_table, int32_t* target_argmax, int32_t* path,
                     int32_t* accept_len, int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot,
                     const ddtree_sampling* sampling, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return accept_launch(target_logits, dtype, V, row_stride, node_token, parent, n_nodes, n_req, L, B, prefix_len,
                       new_prefix_len, k_cache, v_cache, kv, block_table, target_argmax, path, accept_len,
                       next_bonus, src_slot, dst_slot, ws, ws_bytes, stream, sampling);
}

size_t ddtree_lmhead_workspace_bytes(int rows) { return rows < 1 ? 0 : lm_ws_bytes(rows); }

int ddtree_lmhead_argmax(const void* hidden, const void* weight, int rows, int V, int d, int32_t* out_argmax,
                         float* out_max, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int st = lmhead_check(hidden, weight, rows, V, d, out_argmax);
  if (st) return st;
  if (!ws || !aligned16(ws) || ws_bytes < lm_ws_bytes(rows)) return DDTREE_ERR_INVALID_ARG;
  return lmhead_launch(hidden, weight, rows, V, d, out_argmax, out_max, ws, num_sms(), stream, g_attn_wait_ns);
}

int ddtree_walk(const int32_t* target_token, const int32_t* node_token, const int32_t* parent, const int32_t* n_nodes,
                int n_req, int L, int B, const int32_t* prefix_len, int32_t* new_prefix_len, void* k_cache,
                void* v_cache, const ddtree_kv_desc* kv, const int32_t* block_table, int dtype, int32_t* path,
                int32_t* accept_len, int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot, cudaStream_t stream) {
  return walk_launch(target_token, node_token, parent, n_nodes, n_req, L, B, prefix_len, new_prefix_len, k_cache,
                     v_cache, kv, block_table, dtype, path, accept_len, next_bonus, src_slot, dst_slot, stream);
}

size_t ddtree_accept_workspace_bytes(int n_req, int B, int V) {
  (void)V;
  if (n_req < 1 || B < 0) return 0;
  return accept_ws(n_req, B);
}

int ddtree_accept(const void* target_logits, int dtype, int V, long long row_stride, const int32_t* node_token,
                  const int32_t* parent, const int32_t* n_nodes, int n_req, int L, int B,
                  const int32_t* prefix_len, int32_t* new_prefix_len, void* k_cache, void* v_cache,
                  const ddtree_kv_desc* kv, const int32_t* block_table, int32_t* target_argmax, int32_t* path,
                  int32_t* accept_len, int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot, void* ws,
                  size_t ws_bytes, cudaStream_t stream) {
  return accept_launch(target_logits, dtype, V, row_stride, node_token, parent, n_nodes, n_req, L, B,
                       prefix_len, new_prefix_len, k_cache, v_cache, kv, block_table, target_argmax, path,
                       accept_len, next_bonus, src_slot, dst_slot, ws, ws_bytes, stream);
}

static size_t round_parts(const ddtree_round_args* a, size_t* off_attn, size_t* off_acc) {
  const size_t t = align256(topk_ws(a->n_req * a->L, a->V, a->K, a->dtype));
  const size_t at = align256(attn_ws(&a->kv, a->B, a->dtype));
  const size_t ac = a->target_hidden ? align256(lm_ws_bytes(a->n_req * (a->B + 1)) + (size_t)a->n_req * (a->B + 1) * 4)
                                     : align256(accept_ws(a->n_req, a->B));
  if (off_attn) *off_attn = t;
  if (off_acc) *off_acc = t + at;
  return t + at + ac;
}

size_t ddtree_round_workspace_bytes(const ddtree_round_args* a) {
  if (!a || a->n_req < 1 || a->L < 1 || a->V < 1 || a->K < 1 || a->B < 0 || kv_check(&a->kv)) return 0;
  return round_parts(a, nullptr, nullptr);
}

int ddtree_round_launch_count(const ddtree_round_args* a) {
  if (!a || a->n_req < 1 || a->L < 1 || a->V < 1 || a->K < 1 || a->B < 0 || kv_check(&a->kv)) return -1;
  int n = 2;                                                             // top-K, build
  n += 1;                                                                // attention
  if (use_tc_attn(a->dtype, &a->kv) && attn_tc_ws_bytes(geom_of(&a->kv, a->B), num_sms()) > 0) n += 1;   // combine
  if (a->tree_k_in != nullptr) n += 1;                                   // tree K/V write
  if (a->target_hidden != nullptr) return n + 2;                         // LM-head argmax, walk
  n += 1;                                                                // argmax (+ walk)
  if (a->kv.layers > WALK_FUSE_MAX_LAYERS) n += 1;                       // walk and compaction
  return n;
}

// Stage boundaries of a round: an NVTX range per stage on the host timeline
// and, when the caller passes events, one event recorded on the stream at
// each boundary (before top-K, build, tree K/V write, attention, accept, and
// after accept).
struct StageMarks {
  cudaEvent_t* ev;
  cudaStream_t s;
  int i = 0;
  bool open = false;
  int next(const char* name) {
    if (open) nvtxRangePop();
    open = name != nullptr;
    if (open) nvtxRangePushA(name);
    if (ev != nullptr) {
      cudaError_t e = cudaEventRecord(ev[i], s);
      if (e != cudaSuccess) return cuda_fail(e, "ddtree_round: stage event");
    }
    ++i;
    return DDTREE_OK;
  }
  ~StageMarks() {
    if (open) nvtxRangePop();
  }
};

static int round_stages(const ddtree_round_args* a, cudaStream_t stream, char* ws, size_t off_attn, size_t off_acc,
                        size_t need, StageMarks& mk) {
  int st;
  if ((st = mk.next("ddtree_topk"))) return st;
  st = topk_launch(a->drafter_logits, a->dtype, a->n_req * a->L, a->V, a->drafter_stride, a->K, a->ids, a->lp,
                   a->lse, ws, off_attn, stream);
  if (st) return st;
  if ((st = mk.next("ddtree_build"))) return st;
  st = build_launch(a->ids, a->lp, a->root_token, a->n_req, a->L, a->K, a->B, a->node_token, a->parent, a->depth,
                    a->node_rank, a->score, a->anc, a->n_nodes, stream, 0, a->gain_floor, nullptr);
  if (st) return st;
  if ((st = mk.next("ddtree_tree_kv_write"))) return st;
  if (a->tree_k_in != nullptr) {   // the tree's positions are known now: rotate and write its K/V
    st = rope_launch(a->tree_q_in, a->tree_q_in ? (void*)a->q : nullptr, a->tree_k_in, a->tree_v_in, a->dtype,
                     a->depth, a->n_nodes, a->prefix_len, &a->kv, a->block_table, a->B, a->rope_theta, a->k_cache,
                     a->v_cache, stream);
    if (st) return st;
  }
  if ((st = mk.next("ddtree_tree_attn"))) return st;
  // Directly after the build (no RoPE write in between), the attention starts
  // while the build runs: its prefix tiles need no tree (the kernels wait for
  // the build before the tree tiles and the epilogue).
  st = attn_launch(a->q, a->k_cache, a->v_cache, a->dtype, &a->kv, a->block_table, a->prefix_len, a->anc,
                   a->n_nodes, a->B, a->attn_out, a->attn_lse, ws + off_attn, off_acc - off_attn, stream,
                   a->tree_k_in == nullptr ? 1 : 0);
  if (st) return st;
  if ((st = mk.next("ddtree_accept"))) return st;
  if (a->target_hidden != nullptr) {   // the target's argmax from its LM head, logits never written
    if (a->dtype != DDTREE_BF16 || (a->sampling && a->sampling->temperature > 0.0)) return DDTREE_ERR_UNSUPPORTED;
    const int rows = a->n_req * (a->B + 1);
    if ((st = lmhead_check(a->target_hidden, a->lm_head, rows, a->V, a->d_model, a->target_argmax ? a->target_argmax
                                                                                                   : (int32_t*)ws)))
      return st;
    int32_t* tok = a->target_argmax ? a->target_argmax
                                    : (int32_t*)(ws + off_acc + align256(lm_ws_bytes(rows)));
    if ((st = lmhead_launch(a->target_hidden, a->lm_head, rows, a->V, a->d_model, tok, nullptr, ws + off_acc,
                            num_sms(), stream, g_attn_wait_ns)))
      return st;
    st = walk_launch(tok, a->node_token, a->parent, a->n_nodes, a->n_req, a->L, a->B, a->prefix_len,
                     a->new_prefix_len, a->k_cache, a->v_cache, &a->kv, a->block_table, a->dtype, a->path,
                     a->accept_len, a->next_bonus, a->src_slot, a->dst_slot, stream);
  } else {
    st = accept_launch(a->target_logits, a->dtype, a->V, a->target_stride, a->node_token, a->parent, a->n_nodes,
                       a->n_req, a->L, a->B, a->prefix_len, a->new_prefix_len, a->k_cache, a->v_cache, &a->kv,
                       a->block_table, a->target_argmax, a->path, a->accept_len, a->next_bonus, a->src_slot,
                       a->dst_slot, ws + off_acc, need - off_acc, stream, a->sampling);
  }
  if (st) return st;
  return mk.next(nullptr);
}

int ddtree_round(const ddtree_round_args* a, cudaStream_t stream) {
  if (!a) return DDTREE_ERR_INVALID_ARG;
  if (kv_check(&a->kv)) return DDTREE_ERR_INVALID_ARG;
  if (a->kv.n_req != a->n_req) return DDTREE_ERR_INVALID_ARG;
  size_t off_attn = 0, off_acc = 0;
  const size_t need = round_parts(a, &off_attn, &off_acc);
  if (!a->ws || a->ws_bytes < need) return DDTREE_ERR_INVALID_ARG;
  StageMarks mk{a->stage_events, stream};
  return round_stages(a, stream, (char*)a->ws, off_attn, off_acc, need, mk);
}

int ddtree_attn_plan(const ddtree_kv_desc* kv, int B, int dtype, int sms, int* kernel, int* splits) {
  int st = kv_check(kv);
  if (st) return st;
  if (!dtype_ok(dtype) || B < 0 || B > MAX_B || sms < 0 || !kernel || !splits) return DDTREE_ERR_INVALID_ARG;
  if (!use_tc_attn(dtype, kv)) {
    *kernel = 0;
    *splits = 1;
    return DDTREE_OK;
  }
  const AttnDispatch d = attn_dispatch(geom_of(kv, B), sms > 0 ? sms : num_sms());
  *kernel = d.v2 ? 2 : 1;
  *splits = d.v2 ? d.splits : d.v1.splits;
  return DDTREE_OK;
}

int ddtree_debug_attn_timeout(unsigned long long wait_ns, int withhold_tile) {
  if (withhold_tile < -1) return DDTREE_ERR_INVALID_ARG;
  g_attn_wait_ns = wait_ns;
  g_attn_stop_tile = withhold_tile;
  return DDTREE_OK;
}

// ---------------------------------------------------------------- host-buffer round
static int round_host_plan(const ddtree_round_args* a, const ddtree_round_host_io* h, unsigned long long* h2d,
                           unsigned long long* d2h, cudaStream_t s, bool run) {
  if (!a || !h) return DDTREE_ERR_INVALID_ARG;
  if (kv_check(&a->kv) || a->kv.n_req != a->n_req || !dtype_ok(a->dtype)) return DDTREE_ERR_INVALID_ARG;
  const size_t es = (size_t)esize_of(a->dtype);
  const size_t N = (size_t)a->n_req, n = (size_t)a->B + 1, layers = (size_t)a->kv.layers;
  const size_t row = (size_t)a->kv.Hkv * a->kv.D * es;                 // one cache slot
  const size_t qbytes = layers * N * n * a->kv.Hq * a->kv.D * es;
  unsigned long long in = 0, out = 0;
  auto h2d_copy = [&](void* dst, const void* src, size_t bytes) -> int {
    if (!src) return DDTREE_OK;
    if (!dst) return DDTREE_ERR_INVALID_ARG;
    in += bytes;
    if (run && cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return DDTREE_ERR_CUDA;
    return DDTREE_OK;
  };
  auto d2h_copy = [&](void* dst, const void* src, size_t bytes) -> int {
    if (!dst) return DDTREE_OK;
    if (!src) return DDTREE_ERR_INVALID_ARG;
    out += bytes;
    if (run && cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return DDTREE_ERR_CUDA;
    return DDTREE_OK;
  };
  int st;
  if ((st = h2d_copy((void*)a->drafter_logits, h->drafter_logits, N * a->L * (size_t)a->drafter_stride * es))) return st;
  if ((st = h2d_copy((void*)a->root_token, h->root_token, N * 4))) return st;
  if ((st = h2d_copy((void*)a->q, h->q, qbytes))) return st;
  if ((st = h2d_copy((void*)a->target_logits, h->target_logits, N * n * (size_t)a->target_stride * es))) return st;
  if ((st = h2d_copy((void*)a->prefix_len, h->prefix_len, N * 4))) return st;
  if ((h->tree_k != nullptr) != (h->tree_v != nullptr)) return DDTREE_ERR_INVALID_ARG;
  if (h->tree_k) {
    if (!h->prefix_len || !a->k_cache || !a->v_cache) return DDTREE_ERR_INVALID_ARG;
    if (a->kv.paged && !a->block_table) return DDTREE_ERR_INVALID_ARG;
    // a paged cache's block table is device memory: the host cannot address its tree slots
    if (a->kv.paged) return DDTREE_ERR_UNSUPPORTED;
    const size_t cap = (size_t)a->kv.s_max;
    for (size_t r = 0; r < N; ++r) {
      const int P = h->prefix_len[r];
      if (P < 0 || (size_t)P + n > cap) return DDTREE_ERR_INVALID_ARG;
      for (int c = 0; c < 2; ++c) {
        const unsigned char* src = (const unsigned char*)(c ? h->tree_v : h->tree_k) + r * n * row;
        unsigned char* dst = (unsigned char*)(c ? a->v_cache : a->k_cache) + (r * cap + (size_t)P) * row;
        // one 2-D copy over the layers: rows of n * row bytes
        in += layers * n * row;
        if (run && cudaMemcpy2DAsync(dst, N * cap * row, src, N * n * row, n * row, layers, cudaMemcpyHostToDevice,
                                     s) != cudaSuccess)
          return DDTREE_ERR_CUDA;
      }
    }
  }
  if (run && (st = ddtree_round(a, s))) return st;
  if ((st = d2h_copy(h->attn_out, a->attn_out, qbytes))) return st;
  if ((st = d2h_copy(h->node_token, a->node_token, N * n * 4))) return st;
  if ((st = d2h_copy(h->parent, a->parent, N * n * 4))) return st;
  if ((st = d2h_copy(h->n_nodes, a->n_nodes, N * 4))) return st;
  if ((st = d2h_copy(h->path, a->path, N * (a->L + 1) * 4))) return st;
  if ((st = d2h_copy(h->accept_len, a->accept_len, N * 4))) return st;
  if ((st = d2h_copy(h->next_bonus, a->next_bonus, N * 4))) return st;
  if ((st = d2h_copy(h->new_prefix_len, a->new_prefix_len, N * 4))) return st;
  if (h2d) *h2d = in;
  if (d2h) *d2h = out;
  return DDTREE_OK;
}

int ddtree_round_host(const ddtree_round_args* dev, const ddtree_round_host_io* host, cudaStream_t stream) {
  int st = round_host_plan(dev, host, nullptr, nullptr, stream, false);   // validate before any copy
  if (st) return st;
  return round_host_plan(dev, host, nullptr, nullptr, stream, true);
}

int ddtree_round_host_bytes(const ddtree_round_args* dev, const ddtree_round_host_io* host, unsigned long long* h2d,
                            unsigned long long* d2h) {
  return round_host_plan(dev, host, h2d, d2h, nullptr, false) ? -1 : 0;
}

const char* ddtree_status_string(int status) {
  switch (status) {
    case DDTREE_OK: return "ok";
    case DDTREE_ERR_INVALID_ARG: return "invalid argument";
    case DDTREE_ERR_UNSUPPORTED: return "unsupported configuration";
    case DDTREE_ERR_CUDA: return "CUDA error";
    case DDTREE_ERR_NONFINITE: return "non-finite logits";
    case DDTREE_ERR_TIMEOUT: return "bounded wait timed out";
    case DDTREE_ERR_CAPACITY: return "prefix plus tree exceeds the KV cache";
    case DDTREE_ERR_SCRATCH_LIMIT: return "request needs more than the built-in 4 MiB scratch";
    default: return "unknown status";
  }
}

int ddtree_device_status(cudaStream_t stream, unsigned int* bits) {
  if (!bits) return DDTREE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return DDTREE_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return DDTREE_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return DDTREE_ERR_CUDA;
  *bits = v;
  return DDTREE_OK;
}

int ddtree_version(void) { return 200; }

const char* ddtree_last_error(void) { return last_error_buf(); }

}  // extern "C"

// ----------------------------------------------------------------------
// Top-K with built-in scratch, for callers that cannot allocate device
// memory while they run (see ddtree_topk_static_ws in ddtree.h).
// ----------------------------------------------------------------------
namespace {

constexpr size_t STATIC_SCRATCH_BYTES = (size_t)4 << 20;   // 4 MiB per device
constexpr int STATIC_SCRATCH_MAX_DEVICES = 64;

// The scratch array itself.  In host code its name is only a stand-in:
// kernels get the device address looked up below, never the symbol.
__device__ __align__(256) unsigned char g_topk_static_scratch[STATIC_SCRATCH_BYTES];

void* g_static_scratch_ptr[STATIC_SCRATCH_MAX_DEVICES];

// Device address of the scratch array on the current device, looked up once
// per device (nullptr on failure).
void* static_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= STATIC_SCRATCH_MAX_DEVICES) return nullptr;
  if (g_static_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_topk_static_scratch) != cudaSuccess) return nullptr;
    g_static_scratch_ptr[dev] = ptr;
  }
  return g_static_scratch_ptr[dev];
}

}  // namespace

extern "C" {

int ddtree_topk_static_ws(const void* logits, int dtype, int rows, int V, long long row_stride, int K, int32_t* ids,
                          float* lp, float* lse, cudaStream_t stream) {
  int st = topk_check(logits, dtype, rows, V, row_stride, K, ids, lp);
  if (st) return st;
  const TopkPlan p = topk_plan(rows, V, K, esize_of(dtype), num_sms());
  if (p.cpr == 0) return DDTREE_ERR_UNSUPPORTED;
  const size_t need = topk_ws_bytes(rows, p);
  if (need > STATIC_SCRATCH_BYTES) return DDTREE_ERR_SCRATCH_LIMIT;
  void* ws = static_scratch_ptr();
  if (ws == nullptr) return DDTREE_ERR_CUDA;
  // the per-row tickets must start at zero; a previous call normally leaves
  // them at zero, but the array is shared, so clear them every time
  if (cudaMemsetAsync(ws, 0, align256((size_t)rows * 4), stream) != cudaSuccess) return DDTREE_ERR_CUDA;
  return topk_launch(logits, dtype, rows, V, row_stride, K, ids, lp, lse, ws, need, stream);
}

}  // extern "C"
