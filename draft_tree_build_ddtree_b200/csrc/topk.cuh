// Stage 1: per-position log-softmax and top-K over the drafter's block logits.
//
// "DDTree Deep Dive" §1 (per-position marginals q_i from one drafter pass)
// and §2 Lemma 1 (only the top K = min(B, |V|) tokens per position matter).
//
// Design (HBM-bound: every logit is read once, nothing else is large):
//  * A row of V logits is cut into `cpr` chunks; one 512-thread CTA per
//    chunk issues all of its 128-bit loads up front (VPT vectors per
//    thread, a template parameter), so one wave of CTAs keeps the whole
//    input in flight, and stages the chunk in shared memory.  The passes
//    over it are rolled loops over 16-byte vectors, which keeps the kernel's
//    code small enough to stay in the instruction cache (fully unrolled
//    register passes stalled on instruction fetch).
//  * The chunk's sum of exp(z - max) is taken in fp64 so that
//    log q = z - lse, rounded once to fp32, is the correctly rounded value
//    in all but vanishingly rare cases.  exp is a table-driven fp64
//    exponential (Tang's method: 2^(k/64) from a 64-entry table times a
//    degree-5 polynomial of the reduced argument).  bf16 logits sit on a
//    coarse grid, many prefixes tie exactly in real arithmetic, and only a
//    correctly rounded log-prob table orders them reproducibly.
//  * The chunk's threshold value (the K'-th largest logit, K' = min(K,
//    chunk length)) comes, for bf16, from one 256-bin histogram anchored at
//    the chunk maximum: each bin is one bf16 value, so one pass finds it
//    whenever it lies within 256 bf16 steps of the maximum (2 octaves, 13-16%
//    of a Gaussian row).  Otherwise (and for fp32) an 8-bit-digit radix
//    select over the value keys runs.  Every logit >= the threshold is
//    emitted when they fit the chunk's candidate capacity (K + min(K, 512));
//    only then are ties at the threshold cut by lowest token id with a
//    radix select over the complemented index.
//  * The last CTA of the row (atomic ticket, nobody waits) merges the row:
//    combines the chunk sums into lse, selects the top-K among the
//    candidates (unique 64-bit keys: value key, complemented token id),
//    sorts them with a bitonic network and writes ids, lp, lse.
#pragma once

#include "common.cuh"
#include "exp64_table.h"

namespace ddt {

constexpr int TOPK_THREADS = 512;
constexpr int TOPK_MAX_VPT = 6;            // 16-byte vectors per thread
constexpr int TOPK_MAX_CAND = 16384;       // merge capacity (candidates per row)
constexpr int TOPK_MAX_CPR = 128;          // chunks per row
constexpr int TOPK_EXP_WARPS = 6;          // warps of a CTA that sum exp while the others select (4, 5, 7, 8, 10, 12 measured slower)
constexpr int TOPK_LIST_CAP = 4096;        // bf16 candidate list entries per chunk
constexpr int TOPK_MERGE_SMALL = 512;      // merge ranks by counting up to this many keys >= the K-th value
constexpr int TOPK_ID_BITS = 20;           // V <= 2^20
constexpr uint32_t TOPK_ID_MASK = (1u << TOPK_ID_BITS) - 1u;
constexpr int LID_BITS = 15;               // chunk <= 24576 < 32768
constexpr uint32_t LID_MASK = (1u << LID_BITS) - 1u;

struct TopkPlan {
  int cpr;      // chunks per row (0: unsupported)
  int chunk;    // elements per chunk (multiple of the vector width)
  int vpt;      // 16-byte vectors per thread
  int cap;      // candidate slots per chunk
  int cand;     // candidate slots per row = cpr * cap
  int esize;    // bytes per logit
};

inline int topk_cap(int K) { return K + (K < 512 ? K : 512); }

inline TopkPlan topk_plan(int rows, int V, int K, int esize, int num_sms) {
  const int epv = 16 / esize;
  const int max_chunk = TOPK_THREADS * TOPK_MAX_VPT * epv;
  TopkPlan p;
  p.cap = topk_cap(K);
  const int cpr_min = ceil_div(V, max_chunk);
  int cpr = num_sms / (rows > 0 ? rows : 1);
  const int cpr_small = ceil_div(V, 2048);
  if (cpr > cpr_small) cpr = cpr_small;
  int cpr_cap = TOPK_MAX_CAND / p.cap;
  if (cpr_cap > TOPK_MAX_CPR) cpr_cap = TOPK_MAX_CPR;
  if (cpr > cpr_cap) cpr = cpr_cap;
  if (cpr < cpr_min) cpr = cpr_min;
  if (cpr < 1) cpr = 1;
  p.chunk = ceil_div(ceil_div(V, cpr), epv) * epv;
  p.cpr = ceil_div(V, p.chunk);
  p.vpt = ceil_div(ceil_div(p.chunk, epv), TOPK_THREADS);
  p.cand = p.cpr * p.cap;
  p.esize = esize;
  if (p.cpr > cpr_cap || p.vpt > TOPK_MAX_VPT) p.cpr = 0;   // unsupported shape
  return p;
}

// Shared memory of a staged chunk (whole 16-byte vectors), 16-byte aligned.
__host__ __device__ inline size_t topk_stage_bytes(const TopkPlan& p) {
  const size_t v = ((size_t)p.chunk * p.esize + 15) / 16 + 1;
  return v * 16;
}

// Workspace of the top-K stage: tickets, chunk statistics, candidate counts
// and candidates (value key << 20 | complemented token id).
struct TopkWs {
  uint32_t* ticket;          // [rows]
  double2* stats;            // [rows][cpr]: (chunk max, sum of exp(z - max))
  int* count;                // [rows][cpr]
  uint32_t* thr;             // [rows][cpr] the chunk's threshold value key
  unsigned long long* cand;  // [rows][cpr][cap]
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline size_t topk_ws_bytes(int rows, const TopkPlan& p) {
  return align256((size_t)rows * 4) + align256((size_t)rows * p.cpr * 16) + 2 * align256((size_t)rows * p.cpr * 4) +
         align256((size_t)rows * p.cand * 8);
}

inline TopkWs topk_ws_carve(void* ws, int rows, const TopkPlan& p) {
  char* b = (char*)ws;
  TopkWs w;
  w.ticket = (uint32_t*)b;
  b += align256((size_t)rows * 4);
  w.stats = (double2*)b;
  b += align256((size_t)rows * p.cpr * 16);
  w.count = (int*)b;
  b += align256((size_t)rows * p.cpr * 4);
  w.thr = (uint32_t*)b;
  b += align256((size_t)rows * p.cpr * 4);
  w.cand = (unsigned long long*)b;
  return w;
}

// exp(x) in fp64 for -700 <= x <= 700 (table-driven; relative error ~1e-16).
// x is clamped at -700 from below, where exp is ~1e-304 and the result
// stays normal.  The
// reduction k = round(x * 64/ln2) rounds with the 1.5*2^52 shifter (k lands in
// the low word), r = x - k*ln2/64 in two exact-product steps, then
// 2^(k/64) * exp(r) = 2^(k>>6) * T[k&63] * (1 + p(r)).
__device__ __forceinline__ double exp64(double x, const double* tab) {
  x = fmax(x, -700.0);
  const double shifter = 0x1.8p52;
  const double t = fma(x, EXP64_INV_LN2_64, shifter);
  const int k = __double2loint(t);
  const double kd = t - shifter;
  double r = fma(-kd, EXP64_C1, x);
  r = fma(-kd, EXP64_C2, r);
  double p = fma(r, 1.0 / 120.0, 1.0 / 24.0);
  p = fma(p, r, 1.0 / 6.0);
  p = fma(p, r, 0.5);
  p = fma(p, r, 1.0);
  p *= r;                                   // exp(r) - 1
  const double tj = tab[k & 63];
  const double y = fma(tj, p, tj);          // 2^(j/64) * exp(r), in [0.99, 2.02)
  return __hiloint2double(__double2hiint(y) + ((k >> 6) << 20), __double2loint(y));
}

// exp(z) in fp64 for every bf16 bit pattern z with |z| <= 700 (others 0),
// built once per device by exp_bf16_table_kernel.  With it a chunk's sum of
// exp(z - m) is one cached table load and one fp64 add per logit, scaled by
// exp(-m) once: the fp64 exponential, which B200 runs at a small fraction of
// its fp32 rate, is paid per distinct value instead of per logit.
__device__ double g_exp_bf16[65536];

__global__ void exp_bf16_table_kernel() {
  __shared__ double tab[64];
  if (threadIdx.x < 64) tab[threadIdx.x] = EXP64_TABLE[threadIdx.x];
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < 65536) {
    const float z = __uint_as_float((uint32_t)i << 16);
    const double zd = (double)z;
    g_exp_bf16[i] = (z == z && fabs(zd) <= 700.0) ? exp64(zd, tab) : 0.0;
  }
}

// A chunk uses the table when its maximum keeps every scaled sum in range.
constexpr double EXP_TABLE_MAX_M = 600.0;


template <int DT>
struct TopkTraits;
template <>
struct TopkTraits<DDTREE_BF16> {
  static constexpr int EPV = 8;
  static constexpr int KEY_BITS = 16;
};
template <>
struct TopkTraits<DDTREE_F32> {
  static constexpr int EPV = 4;
  static constexpr int KEY_BITS = 32;
};

template <int DT>
__device__ __forceinline__ uint32_t elem_bits(const uint4& v, int j) {
  if (DT == DDTREE_BF16) return (u32_at(v, j >> 1) >> (16 * (j & 1))) & 0xFFFFu;
  return u32_at(v, j);
}
template <int DT>
__device__ __forceinline__ uint32_t value_key(uint32_t bits) {
  return DT == DDTREE_BF16 ? key16_of_bf16((uint16_t)bits) : key32_of_f32(__uint_as_float(bits));
}
template <int DT>
__device__ __forceinline__ float key_value(uint32_t key) {
  return DT == DDTREE_BF16 ? bf16_of_key16(key) : f32_of_key32(key);
}

// Warp-aggregated append of `key` to dst[*counter] where `take` holds; every
// lane of the warp calls it.
__device__ __forceinline__ void append_to(unsigned long long* dst, int* counter, bool take, unsigned long long key,
                                          int lane) {
  const unsigned bal = __ballot_sync(0xffffffffu, take);
  if (bal) {
    int base = 0;
    if (lane == 0) base = atomicAdd(counter, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) dst[base + __popc(bal & ((1u << lane) - 1u))] = key;
  }
}

template <int DT, int VPT>
__global__ void __launch_bounds__(TOPK_THREADS, 1)
topk_kernel(const void* __restrict__ logits, int rows, int V, long long row_stride, int K, TopkPlan plan,
            TopkWs ws, int32_t* __restrict__ out_ids, float* __restrict__ out_lp, float* __restrict__ out_lse) {
  typedef TopkTraits<DT> T;
  constexpr int EPV = T::EPV;
  constexpr int NW = TOPK_THREADS / 32;
  constexpr int NWE = TOPK_EXP_WARPS;                 // warps 0..NWE-1: exp-sum; the rest: selection
  constexpr int SEL_THREADS = TOPK_THREADS - 32 * NWE;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ uint32_t hist[256];
  __shared__ int bcast[4];
  __shared__ uint32_t red_u[NW];
  __shared__ uint32_t red_w[NW];
  __shared__ double red_d[NWE];
  __shared__ double s_tab[64];
  __shared__ int s_count;
  __shared__ int s_ncl;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x / plan.cpr;
  const int c = blockIdx.x - row * plan.cpr;
  const long long c0 = (long long)c * plan.chunk;
  const int len = (int)min((long long)plan.chunk, (long long)V - c0);
  const int kloc = K < len ? K : len;
  if (tid < 64) s_tab[tid] = EXP64_TABLE[tid];
  for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0;
  if (tid == 0) { s_count = 0; s_ncl = 0; }

  // ---- streaming load: every vector of this thread in flight at once; the
  //      thread maximum is taken from the registers, then the chunk is staged ----
  const unsigned char* base = (const unsigned char*)logits + ((long long)row * row_stride + c0) * (16 / EPV);
  const int nvec_full = len / EPV;
  const int tail = len - nvec_full * EPV;          // ragged end (V not a multiple of the vector width)
  const int nvec = nvec_full + (tail > 0 ? 1 : 0);
  uint4* chunk_s = reinterpret_cast<uint4*>(smem_raw);
  // candidate list of the selection warps (bf16): value key << 16 | chunk-local index
  uint32_t* clist = reinterpret_cast<uint32_t*>(smem_raw + topk_stage_bytes(plan));
  // bf16: fp32 max of the widened halves (fmaxf skips NaN, the magnitude maxima
  // detect it); fp32: max of the order keys.  tkey: the thread maximum's key.
  float mx = -INFINITY;
  uint32_t tkey = 0, mag = 0;
  bool nan_seen = false;
  auto take_vec = [&](const uint4& v, int valid) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w = u32_at(v, q);
      if (DT == DDTREE_BF16) {
        const float lo = 2 * q < valid ? __uint_as_float(w << 16) : -INFINITY;
        const float hi = 2 * q + 1 < valid ? __uint_as_float(w & 0xFFFF0000u) : -INFINITY;
        mx = fmaxf(mx, fmaxf(lo, hi));
        if (2 * q < valid) mag = max(mag, w & 0x7FFFu);
        if (2 * q + 1 < valid) mag = max(mag, (w >> 16) & 0x7FFFu);
      } else if (q < valid) {
        const float f = __uint_as_float(w);
        nan_seen |= f != f;
        tkey = max(tkey, key32_of_f32(f));
      }
    }
  };
  {
    uint4 vec[VPT];
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int vi = v * TOPK_THREADS + tid;
      vec[v] = vi < nvec_full ? ldg_stream_v4(base + (size_t)vi * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int vi = v * TOPK_THREADS + tid;
      if (vi < nvec_full) {
        take_vec(vec[v], EPV);
        chunk_s[vi] = vec[v];
      }
    }
  }
  if (tail > 0 && tid == 0) {
    uint4 tv = make_uint4(0u, 0u, 0u, 0u);
    for (int j = 0; j < tail; ++j) {
      uint32_t x;
      int q;
      if (DT == DDTREE_BF16) {
        x = (uint32_t)((const uint16_t*)(base + (size_t)nvec_full * 16))[j] << (16 * (j & 1));
        q = j >> 1;
      } else {
        x = ((const uint32_t*)(base + (size_t)nvec_full * 16))[j];
        q = j;
      }
      if (q == 0) tv.x |= x; else if (q == 1) tv.y |= x; else if (q == 2) tv.z |= x; else tv.w |= x;
    }
    take_vec(tv, tail);
    chunk_s[nvec_full] = tv;
  }
  if (DT == DDTREE_BF16) {
    nan_seen = mag > 0x7F80u;
    tkey = mx > -INFINITY ? key32_of_f32(mx) >> 16 : 0u;
  }

  // Element e of vector vi is logit c0 + vi*EPV + e; its order key is 0 past the chunk end.
  // bf16 keys are computed two at a time with 16-bit SIMD integer ops.
  auto keys_of = [&](int vi, uint32_t* k) {
    const uint4 v = chunk_s[vi];
    const int valid = len - vi * EPV;              // >= EPV except in the ragged last vector
    if (DT == DDTREE_BF16) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t k2 = key16x2_of_bf16x2(u32_at(v, q));
        k[2 * q] = (2 * q < valid) ? (k2 & 0xFFFFu) : 0u;
        k[2 * q + 1] = (2 * q + 1 < valid) ? (k2 >> 16) : 0u;
      }
    } else {
#pragma unroll
      for (int j = 0; j < EPV; ++j) k[j] = (j < valid) ? key32_of_f32(__uint_as_float(u32_at(v, j))) : 0u;
    }
  };

  // ---- chunk maximum; bf16: lower bound of the K'-th largest logit ----
  if (__any_sync(0xffffffffu, nan_seen) && lane == 0) flag_status(DDTREE_STATUS_NONFINITE);
  if (DT == DDTREE_BF16) {
    // The thread maxima are distinct elements, so if every warp contributes
    // its r-th largest thread maximum (r = ceil(K'/warps)), at least K'
    // logits are >= the smallest of those.  Only logits above that bound
    // enter the window histogram and the candidate list.
    const int r = (kloc + NW - 1) / NW;
    uint32_t wk = 0;
    if (r <= 32) {
      uint32_t x = tkey;                        // 0: none
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {       // bitonic sort across the warp, descending
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
          const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
          const bool lower = (lane & j) == 0;
          const bool desc = (lane & k) == 0 || k == 32;
          x = (lower == desc) ? max(x, y) : min(x, y);
        }
      }
      wk = __shfl_sync(0xffffffffu, x, r - 1);
    }
    if (lane == 0) red_w[warp] = wk;
  }
  uint32_t kmax = __reduce_max_sync(0xffffffffu, tkey);
  if (lane == 0) red_u[warp] = kmax;
  __syncthreads();
  kmax = red_u[0];
#pragma unroll
  for (int i = 1; i < NW; ++i) kmax = red_u[i] > kmax ? red_u[i] : kmax;
  const float m = key_value<DT>(kmax);
  const double md = (double)m;
  const bool m_finite = m > -INFINITY;
  const bool use_table = DT == DDTREE_BF16 && md <= EXP_TABLE_MAX_M && md >= -EXP_TABLE_MAX_M;

  uint32_t tval = 0;
  int above = 0, eq = 0;
  if (warp < NWE) {
    // ================= exp warps: fp64 sum of exp(z - m) =================
    double s0 = 0.0, s1 = 0.0;
    if (m_finite) {
      for (int vi = tid; vi < nvec; vi += 32 * NWE) {
        const uint4 v = chunk_s[vi];
        const int valid = len - vi * EPV;
        // branch-free over the vector (the exps are independent chains); the
        // past-the-end elements of the ragged vector are computed and dropped
        double e[EPV];
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
          if (use_table) {
            e[j] = j < valid ? __ldg(&g_exp_bf16[elem_bits<DT>(v, j)]) : 0.0;   // exp(z); scaled below
          } else {
            const float z = DT == DDTREE_BF16 ? bf16_bits_to_f32((uint16_t)elem_bits<DT>(v, j))
                                              : __uint_as_float(u32_at(v, j));
            e[j] = exp64((double)z - md, s_tab);
            e[j] = j < valid ? e[j] : 0.0;
          }
        }
#pragma unroll
        for (int j = 0; j < EPV; j += 2) { s0 += e[j]; s1 += e[j + 1]; }
      }
    }
    double sum = s0 + s1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) red_d[warp] = sum;
  } else {
    // ================= selection warps: threshold and emission =================
    const int gtid = tid - 32 * NWE;
    auto gsync = [] { named_sync(1, SEL_THREADS); };
    bool found = false, use_list = false;
    if (DT == DDTREE_BF16) {
      // max-anchored window histogram (bin b: the value kmax - b) of the logits
      // above the bound; the same logits enter the candidate list
      uint32_t wbound = red_w[0];
#pragma unroll
      for (int i = 1; i < NW; ++i) wbound = red_w[i] < wbound ? red_w[i] : wbound;
      const uint32_t wkey = max(wbound, kmax >= 255u ? kmax - 255u : 0u);
      const float wlow = wkey > 0u ? bf16_of_key16(wkey) : -INFINITY;
      for (int vi = gtid; vi < nvec; vi += SEL_THREADS) {
        const uint4 v = chunk_s[vi];
        const int valid = len - vi * EPV;
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
          const uint32_t bits = elem_bits<DT>(v, j);
          if (j < valid && bf16_bits_to_f32((uint16_t)bits) >= wlow) {
            const uint32_t key = key16_of_bf16((uint16_t)bits);
            const uint32_t d = kmax - key;
            if (d < 256u) atomicAdd(&hist[d], 1u);
            const int slot = atomicAdd(&s_ncl, 1);
            if (slot < TOPK_LIST_CAP) clist[slot] = (key << 16) | (uint32_t)(vi * EPV + j);
          }
        }
      }
      gsync();
      if (gtid < 32) {
        uint32_t cbin[8];
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { cbin[j] = hist[8 * gtid + j]; mine += cbin[j]; }
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (gtid >= o) incl += v;
        }
        const uint32_t before = incl - mine;
        const unsigned msk = __ballot_sync(0xffffffffu, before < (uint32_t)kloc && (uint32_t)kloc <= incl);
        if (gtid == 0) bcast[3] = msk ? 1 : 0;
        if (msk && gtid == __ffs(msk) - 1) {
          uint32_t acc = before, cb = cbin[0];
          int j0 = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (acc + cbin[j] >= (uint32_t)kloc) { j0 = j; cb = cbin[j]; break; }
            acc += cbin[j];
          }
          bcast[0] = 8 * gtid + j0;
          bcast[1] = (int)acc;
          bcast[2] = (int)cb;
        }
      }
      gsync();
      if (bcast[3]) {
        found = true;
        tval = kmax - (uint32_t)bcast[0];
        above = bcast[1];
        eq = bcast[2];
      }
      // every logit >= the threshold is in the list when it did not overflow
      use_list = found && s_ncl <= TOPK_LIST_CAP;
      gsync();
    }
    if (!found) {
      auto each = [&](auto f) {
        for (int vi = gtid; vi < nvec; vi += SEL_THREADS) {
          uint32_t k[EPV];
          keys_of(vi, k);
#pragma unroll
          for (int j = 0; j < EPV; ++j) f(k[j]);
        }
      };
      const RadixOut<uint32_t> ro = radix_kth_g<uint32_t>(each, T::KEY_BITS, kloc, hist, bcast, gtid, SEL_THREADS, gsync);
      tval = ro.t;
      above = ro.above;
      eq = ro.eq;
    }
    const int ncl = use_list ? s_ncl : 0;

    // ---- emit candidates: every key >= tval, or cut the ties at tval by lowest id ----
    const bool all_ties = above + eq <= plan.cap;
    uint32_t lid_thr = 0;
    if (!all_ties) {
      auto each_lid = [&](auto f) {
        if (use_list) {
          for (int i = gtid; i < ncl; i += SEL_THREADS) {
            const uint32_t e = clist[i];
            f((e >> 16) == tval ? (LID_MASK - (e & 0xFFFFu)) : 0u);
          }
        } else {
          for (int vi = gtid; vi < nvec; vi += SEL_THREADS) {
            uint32_t k[EPV];
            keys_of(vi, k);
#pragma unroll
            for (int j = 0; j < EPV; ++j) f(k[j] == tval ? (LID_MASK - (uint32_t)(vi * EPV + j)) : 0u);
          }
        }
      };
      lid_thr = radix_kth_g<uint32_t>(each_lid, LID_BITS, kloc - above, hist, bcast, gtid, SEL_THREADS, gsync).t;
    }
    unsigned long long* cand = ws.cand + (size_t)row * plan.cand + (size_t)c * plan.cap;
    auto emit = [&](uint32_t key, uint32_t lid) {
      const bool take = key != 0 && (key > tval || (key == tval && (all_ties || (LID_MASK - lid) >= lid_thr)));
      if (take) {
        const int slot = atomicAdd(&s_count, 1);
        const uint32_t gid = (uint32_t)(c0 + lid);
        if (slot < plan.cap)
          cand[slot] = ((unsigned long long)key << TOPK_ID_BITS) | (unsigned long long)(TOPK_ID_MASK - gid);
      }
    };
    if (use_list) {
      for (int i = gtid; i < ncl; i += SEL_THREADS) {
        const uint32_t e = clist[i];
        emit(e >> 16, e & 0xFFFFu);
      }
    } else {
      for (int vi = gtid; vi < nvec; vi += SEL_THREADS) {
        uint32_t k[EPV];
        keys_of(vi, k);
#pragma unroll
        for (int j = 0; j < EPV; ++j) emit(k[j], (uint32_t)(vi * EPV + j));
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    double tot = 0.0;
    for (int i = 0; i < NWE; ++i) tot += red_d[i];
    if (use_table) tot *= exp64(-md, s_tab);           // sum of exp(z) -> sum of exp(z - m)
    ws.stats[(size_t)row * plan.cpr + c] = make_double2(md, tot);
    ws.count[(size_t)row * plan.cpr + c] = s_count < plan.cap ? s_count : plan.cap;
    ws.thr[(size_t)row * plan.cpr + c] = tval;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(&ws.ticket[row], 1u);
    s_last = (t == (unsigned)(plan.cpr - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // =================== merge (last CTA of this row; the staged chunk is dead) ===================
  const unsigned long long* cand_row = ws.cand + (size_t)row * plan.cand;
  unsigned long long* sc = (unsigned long long*)smem_raw;   // [plan.cand]
  int kpow = 1;
  while (kpow < K) kpow <<= 1;
  unsigned long long* win = sc + plan.cand;                 // [max(kpow, TOPK_MERGE_SMALL)]
  __shared__ int s_cnt[TOPK_MAX_CPR];
  __shared__ double2 s_st[TOPK_MAX_CPR];
  __shared__ double s_lse;
  __shared__ int s_m;
  // One round of loads: the chunks' counts, statistics and thresholds, and
  // (speculatively, before the counts are known) the first candidate slots.
  constexpr int UNR = 4;
  const int slots = plan.cpr * plan.cap;
  unsigned long long v[UNR];
#pragma unroll
  for (int u = 0; u < UNR; ++u) {
    const int sl = tid + u * TOPK_THREADS;
    v[u] = sl < slots ? __ldcg(cand_row + sl) : 0ull;
  }
  // Every chunk emitted at least min(K, its length) logits at or above its
  // threshold value, so the row's K-th best value is at least the largest
  // chunk threshold: candidates below it cannot be selected.
  uint32_t tmax = 0;
  for (int i = tid; i < plan.cpr; i += TOPK_THREADS) {
    s_cnt[i] = __ldcg(&ws.count[(size_t)row * plan.cpr + i]);
    s_st[i] = __ldcg(&ws.stats[(size_t)row * plan.cpr + i]);
    const int li = (int)min((long long)plan.chunk, (long long)V - (long long)i * plan.chunk);
    if (li >= K) tmax = max(tmax, __ldcg(&ws.thr[(size_t)row * plan.cpr + i]));
  }
  tmax = __reduce_max_sync(0xffffffffu, tmax);
  if (lane == 0) red_u[warp] = tmax;
  if (tid == 0) { s_count = 0; s_m = 0; }
  __syncthreads();
  uint32_t floor_v = red_u[0];
#pragma unroll
  for (int i = 1; i < NW; ++i) floor_v = red_u[i] > floor_v ? red_u[i] : floor_v;
  const unsigned long long floor_key = (unsigned long long)floor_v << TOPK_ID_BITS;
  // gather the candidates at or above the floor (one shared atomic per warp and round)
  auto append = [&](bool take, unsigned long long key) {
    const unsigned bal = __ballot_sync(0xffffffffu, take);
    if (bal) {
      int base = 0;
      if (lane == 0) base = atomicAdd(&s_count, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (take) sc[base + __popc(bal & ((1u << lane) - 1u))] = key;
    }
  };
#pragma unroll
  for (int u = 0; u < UNR; ++u) {
    const int sl = tid + u * TOPK_THREADS;
    const int ci = sl / plan.cap, j = sl - ci * plan.cap;
    append(sl < slots && j < s_cnt[ci] && v[u] >= floor_key, v[u]);
  }
  for (int s0 = UNR * TOPK_THREADS + (tid & ~31); s0 < slots; s0 += UNR * TOPK_THREADS) {   // warp-uniform
    unsigned long long w[UNR];
    bool ok[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int sl = s0 + lane + u * TOPK_THREADS;
      const int ci = sl / plan.cap, j = sl - ci * plan.cap;
      ok[u] = sl < slots && j < s_cnt[ci];
      w[u] = ok[u] ? __ldcg(cand_row + sl) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) append(ok[u] && w[u] >= floor_key, w[u]);
  }
  if (warp == NW - 1) {   // lse from the chunk statistics, combined across the lanes of the last warp
    double M = -INFINITY;
    for (int i = lane; i < plan.cpr; i += 32) M = fmax(M, s_st[i].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmax(M, __shfl_xor_sync(0xffffffffu, M, o));
    double S = 0.0;
    if (M > -INFINITY)
      for (int i = lane; i < plan.cpr; i += 32)
        if (s_st[i].x > -INFINITY) S += s_st[i].y * exp64(s_st[i].x - M, s_tab);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);   // same value on every lane
    if (lane == 0) {
      s_lse = M + log(S);
      ws.ticket[row] = 0;   // leave the workspace ready for the next call
      // order key of the row maximum (the largest chunk maximum)
      bcast[3] = M > -INFINITY ? (int)value_key<DT>(DT == DDTREE_BF16 ? (uint32_t)(__float_as_uint((float)M) >> 16)
                                                                     : __float_as_uint((float)M))
                               : 0;
    }
  }
  __syncthreads();
  const int ncand = s_count;   // <= plan.cand: every chunk wrote at most cap slots
  const double lse = s_lse;
  const uint32_t vkmax = (uint32_t)bcast[3];
  const int per = (ncand + TOPK_THREADS - 1) / TOPK_THREADS;
  // The K-th largest value among the candidates: every key above it and the
  // ties at it form the set that holds the row's top K.  bf16: one
  // max-anchored 256-bin histogram when the value lies within 256 steps of
  // the row maximum, else a radix select.
  RadixOut<uint32_t> vt{0u, 0, 0};
  bool vfound = false;
  if (DT == DDTREE_BF16) {
    for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < ncand; i += TOPK_THREADS) {
      const uint32_t d = vkmax - (uint32_t)(sc[i] >> TOPK_ID_BITS);
      if (d < 256u) atomicAdd(&hist[d], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t cbin[8];
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cbin[j] = hist[8 * lane + j]; mine += cbin[j]; }
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t before = incl - mine;
      const unsigned msk = __ballot_sync(0xffffffffu, before < (uint32_t)K && (uint32_t)K <= incl);
      if (lane == 0) bcast[3] = msk ? 1 : 0;
      if (msk && lane == __ffs(msk) - 1) {
        uint32_t acc = before, cb = cbin[0];
        int j0 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + cbin[j] >= (uint32_t)K) { j0 = j; cb = cbin[j]; break; }
          acc += cbin[j];
        }
        bcast[0] = 8 * lane + j0;
        bcast[1] = (int)acc;
        bcast[2] = (int)cb;
      }
    }
    __syncthreads();
    if (bcast[3]) {
      vfound = true;
      vt = RadixOut<uint32_t>{vkmax - (uint32_t)bcast[0], bcast[1], bcast[2]};
    }
    __syncthreads();
  }
  if (!vfound) {
    auto veach = [&](auto f) {
      for (int i = 0; i < per; ++i) {
        const int idx = i * TOPK_THREADS + tid;
        f(idx < ncand ? (uint32_t)(sc[idx] >> TOPK_ID_BITS) : 0u);
      }
    };
    vt = radix_kth<uint32_t>(veach, T::KEY_BITS, K, hist, bcast);
  }
  const int nsel = vt.above + vt.eq;
  if (nsel <= TOPK_MERGE_SMALL) {
    for (int i0 = 0; i0 < ncand; i0 += TOPK_THREADS) {   // block-uniform trip count
      const int idx = i0 + tid;
      const unsigned long long k = idx < ncand ? sc[idx] : 0ull;
      append_to(win, &s_m, idx < ncand && (uint32_t)(k >> TOPK_ID_BITS) >= vt.t, k, lane);
    }
    __syncthreads();
    // rank by counting (keys are unique): g threads share one key's count
    int g = 32;
    while (g > 1 && nsel * g > TOPK_THREADS) g >>= 1;
    const int q = tid / g, part = tid - q * g;
    unsigned long long k = 0ull;
    int rank = 0;
    if (q < nsel) {
      k = win[q];
      int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
      int j = part;
      for (; j + 3 * g < nsel; j += 4 * g) {
        r0 += win[j] > k;
        r1 += win[j + g] > k;
        r2 += win[j + 2 * g] > k;
        r3 += win[j + 3 * g] > k;
      }
      for (; j < nsel; j += g) r0 += win[j] > k;
      rank = (r0 + r1) + (r2 + r3);
    }
    for (int o = g >> 1; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (q < nsel && part == 0 && rank < K) {
      const uint32_t vkey = (uint32_t)(k >> TOPK_ID_BITS);
      out_ids[(size_t)row * K + rank] = (int)(TOPK_ID_MASK - (uint32_t)(k & TOPK_ID_MASK));
      out_lp[(size_t)row * K + rank] = (float)((double)key_value<DT>(vkey) - lse);   // one rounding of the fp64 value
    }
    if (out_lse != nullptr && tid == 0) out_lse[row] = (float)lse;
    return;
  }
  // many ties at the K-th value: radix select of the top K keys, then a bitonic sort
  if (tid == 0) s_count = 0;
  __syncthreads();
  auto geach = [&](auto f) {
    for (int i = 0; i < per; ++i) {
      const int idx = i * TOPK_THREADS + tid;
      f(idx < ncand ? sc[idx] : 0ull);
    }
  };
  const unsigned long long gt =
      radix_kth<unsigned long long>(geach, T::KEY_BITS + TOPK_ID_BITS, K, hist, bcast).t;
  for (int i = 0; i < per; ++i) {
    const int idx = i * TOPK_THREADS + tid;
    const unsigned long long k = idx < ncand ? sc[idx] : 0ull;
    if (k != 0 && k >= gt) {
      const int slot = atomicAdd(&s_count, 1);
      if (slot < kpow) win[slot] = k;
    }
  }
  __syncthreads();
  for (int size = 2; size <= kpow; size <<= 1) {     // bitonic sort, descending
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < kpow / 2; i += TOPK_THREADS) {
        const int lo = 2 * stride * (i / stride) + (i % stride);
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const unsigned long long a = win[lo], b = win[hi];
        if ((a < b) == desc) { win[lo] = b; win[hi] = a; }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < K; i += TOPK_THREADS) {
    const unsigned long long k = win[i];
    const uint32_t vkey = (uint32_t)(k >> TOPK_ID_BITS);
    out_ids[(size_t)row * K + i] = (int)(TOPK_ID_MASK - (uint32_t)(k & TOPK_ID_MASK));
    out_lp[(size_t)row * K + i] = (float)((double)key_value<DT>(vkey) - lse);   // one rounding of the fp64 value
  }
  if (out_lse != nullptr && tid == 0) out_lse[row] = (float)lse;
}

inline size_t topk_smem_bytes(const TopkPlan& p, int K) {
  int kpow = 1;
  while (kpow < K) kpow <<= 1;
  const size_t merge = (size_t)(p.cand + (kpow > TOPK_MERGE_SMALL ? kpow : TOPK_MERGE_SMALL)) * 8;
  const size_t chunk = topk_stage_bytes(p) + (size_t)TOPK_LIST_CAP * 4;   // staged chunk + candidate list
  return merge > chunk ? merge : chunk;
}

}  // namespace ddt
