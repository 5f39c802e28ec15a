// Stage 1: per-position log-softmax and top-K over the drafter's block logits.
//
// "DDTree Deep Dive" §1 (per-position marginals q_i from one drafter pass)
// and §2 Lemma 1 (only the top K = min(B, |V|) tokens per position matter).
//
// Design (HBM-bound: every logit is read once, nothing else is large):
//  * A row of V logits is cut into `cpr` chunks; one 512-thread CTA per
//    chunk issues all of its 128-bit loads up front into registers (at most
//    6 vectors per thread), so one wave of CTAs keeps the whole input in
//    flight.
//  * Each CTA reduces its chunk to (max, sum exp(z - max)) and to its local
//    top-K' (K' = min(K, chunk length)).  The sum is taken in fp64 (fp64
//    exp and adds) so that log q = z - lse, rounded once to fp32, is the
//    correctly rounded value in all but vanishingly rare cases: bf16 logits
//    sit on a coarse grid, many prefixes tie exactly in real arithmetic, and
//    only a correctly rounded log-prob table orders them reproducibly.  The
//    local top-K' comes from a radix select on a unique
//    composite key (order key of the logit, then the complemented local
//    index so that lower ids win ties).  For bf16 the first pass is a
//    256-bin histogram anchored at the chunk maximum: each bin is one bf16
//    value, so one pass finds the threshold value whenever the K'-th best
//    logit lies within 256 bf16 steps of the maximum; otherwise the generic
//    8-bit-digit radix select runs.
//  * The candidates go to the workspace; the last CTA of the row (atomic
//    ticket, nobody waits) merges the row: combines the chunk sums into lse,
//    selects the global top-K among the candidates with the same radix
//    select, sorts them with a bitonic network and writes ids, lp, lse.
#pragma once

#include "common.cuh"

namespace ddt {

constexpr int TOPK_THREADS = 512;
constexpr int TOPK_MAX_VPT = 6;            // 16-byte vectors per thread
constexpr int TOPK_MAX_CAND = 16384;       // merge capacity (candidates per row)
constexpr int TOPK_ID_BITS = 20;           // V <= 2^20
constexpr uint32_t TOPK_ID_MASK = (1u << TOPK_ID_BITS) - 1u;

struct TopkPlan {
  int cpr;      // chunks per row
  int chunk;    // elements per chunk (multiple of the vector width)
  int kmax;     // candidates per chunk = min(K, chunk)
  int cand;     // candidates per row
};

inline TopkPlan topk_plan(int rows, int V, int K, int esize, int num_sms) {
  const int epv = 16 / esize;
  const int max_chunk = TOPK_THREADS * TOPK_MAX_VPT * epv;
  int cpr_min = ceil_div(V, max_chunk);
  int cpr_fill = num_sms / (rows > 0 ? rows : 1);
  if (cpr_fill < 1) cpr_fill = 1;
  int cpr_small = ceil_div(V, 2048);
  int cpr = cpr_fill < cpr_small ? cpr_fill : cpr_small;
  if (cpr < cpr_min) cpr = cpr_min;
  int chunk = ceil_div(ceil_div(V, cpr), epv) * epv;
  cpr = ceil_div(V, chunk);
  TopkPlan p;
  p.cpr = cpr;
  p.chunk = chunk;
  p.kmax = K < chunk ? K : chunk;
  // all chunks but the last hold `chunk` elements; the last one may be short
  int last = V - (cpr - 1) * chunk;
  p.cand = (cpr - 1) * p.kmax + (K < last ? K : last);
  return p;
}

// Workspace of the top-K stage, per row: [ticket u32] ... then per chunk
// (max, sumexp) float2, then the candidates (u64).
struct TopkWs {
  uint32_t* ticket;        // [rows]
  double2* stats;          // [rows][cpr]: (chunk max, sum of exp(z - max)) in fp64
  unsigned long long* cand;  // [rows][cand]
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline size_t topk_ws_bytes(int rows, const TopkPlan& p) {
  return align256((size_t)rows * 4) + align256((size_t)rows * p.cpr * 16) +
         align256((size_t)rows * p.cand * 8);
}

inline TopkWs topk_ws_carve(void* ws, int rows, const TopkPlan& p) {
  char* b = (char*)ws;
  TopkWs w;
  w.ticket = (uint32_t*)b;
  b += align256((size_t)rows * 4);
  w.stats = (double2*)b;
  b += align256((size_t)rows * p.cpr * 16);
  w.cand = (unsigned long long*)b;
  return w;
}

// ---------------------------------------------------------------------------
// Block-wide radix select over unique keys.
//
// Keys hold `shift_done` undetermined low bits below an already fixed
// `prefix`; `need` of the keys that share that prefix must be selected (the
// keys above the prefix are selected already).  Returns the threshold t: the
// selection is every key >= t.  `each(f)` calls f(key) for every key this
// thread holds (0 = empty slot), so the caller controls unrolling.
// ---------------------------------------------------------------------------
template <typename KeyT, typename Each>
__device__ __forceinline__ KeyT radix_select(Each each, int shift_done, KeyT prefix, int need,
                                             uint32_t* hist /*[256]*/, int* bcast /*[4]*/) {
  const int tid = threadIdx.x;
  int shift = shift_done;
  while (shift > 0) {
    const int width = shift < 8 ? shift : 8;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int hi = shift + width;
    const KeyT want = (hi >= (int)(8 * sizeof(KeyT))) ? (KeyT)0 : (prefix >> hi);
    each([&](KeyT k) {
      const KeyT top = (hi >= (int)(8 * sizeof(KeyT))) ? (KeyT)0 : (k >> hi);
      if (k != 0 && top == want) atomicAdd(&hist[(uint32_t)(k >> shift) & dmask], 1u);
    });
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits [8l, 8l+8); find digit d with above(d) < need <= above(d) + hist[d]
      uint32_t c[8];
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[8 * tid + j]; mine += c[j]; }
      uint32_t incl = mine;   // suffix sum over lanes: keys in digits >= 8*lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (tid + o < 32) incl += v;
      }
      const uint32_t above_lane = incl - mine;
      const bool here = above_lane < (uint32_t)need && (uint32_t)need <= incl;
      const unsigned m = __ballot_sync(0xffffffffu, here);
      if (tid == __ffs(m) - 1) {
        uint32_t above = above_lane;
        int d = 7;
        for (; d > 0; --d) {
          if (above + c[d] >= (uint32_t)need) break;
          above += c[d];
        }
        bcast[0] = 8 * tid + d;
        bcast[1] = need - (int)above;
        bcast[2] = (int)c[d];
      }
    }
    __syncthreads();
    const int digit = bcast[0];
    need = bcast[1];
    const int cnt = bcast[2];
    __syncthreads();
    prefix |= ((KeyT)digit) << shift;
    if (cnt == need) break;   // every key with this prefix is selected
  }
  return prefix;
}

// ---------------------------------------------------------------------------
// The chunk kernel (+ merge in the last CTA of each row).
// ---------------------------------------------------------------------------
template <int DT>  // DDTREE_BF16 or DDTREE_F32
struct TopkTraits;
template <>
struct TopkTraits<DDTREE_BF16> {
  typedef uint32_t LKey;                 // local composite key16 << 15 | ~lid
  static constexpr int EPV = 8;
  static constexpr int KEY_BITS = 16;
};
template <>
struct TopkTraits<DDTREE_F32> {
  typedef unsigned long long LKey;       // key32 << 15 | ~lid
  static constexpr int EPV = 4;
  static constexpr int KEY_BITS = 32;
};

constexpr int LID_BITS = 15;             // chunk <= 24576 < 32768
constexpr uint32_t LID_MASK = (1u << LID_BITS) - 1u;

template <int DT>
__global__ void __launch_bounds__(TOPK_THREADS)
topk_kernel(const void* __restrict__ logits, int rows, int V, long long row_stride, int K,
            TopkPlan plan, TopkWs ws, int32_t* __restrict__ out_ids, float* __restrict__ out_lp,
            float* __restrict__ out_lse) {
  typedef TopkTraits<DT> T;
  typedef typename T::LKey LKey;
  constexpr int EPV = T::EPV;
  constexpr int E = TOPK_MAX_VPT * EPV;   // elements per thread (max)

  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ uint32_t hist[256];
  __shared__ int bcast[4];
  __shared__ double red_d[TOPK_THREADS / 32];
  __shared__ LKey red_k[TOPK_THREADS / 32];
  __shared__ int s_count;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int row = blockIdx.x / plan.cpr;
  const int c = blockIdx.x - row * plan.cpr;
  const long long c0 = (long long)c * plan.chunk;
  const int len = (int)min((long long)plan.chunk, (long long)V - c0);
  const int kloc = K < len ? K : len;

  // ---- streaming load: all vectors of this thread in flight at once ----
  const unsigned char* base =
      (const unsigned char*)logits + ((long long)row * row_stride + c0) * (16 / EPV);
  const int nvec_full = len / EPV;
  uint4 vec[TOPK_MAX_VPT];
#pragma unroll
  for (int v = 0; v < TOPK_MAX_VPT; ++v) {
    int vi = v * TOPK_THREADS + tid;
    if (vi < nvec_full) vec[v] = ldg_stream_v4(base + (size_t)vi * 16);
    else vec[v] = make_uint4(0, 0, 0, 0);
  }
  // partial tail vector (only when V is not a multiple of the vector width)
  const int tail = len - nvec_full * EPV;
  if (tail > 0 && (nvec_full % TOPK_THREADS) == tid && nvec_full / TOPK_THREADS < TOPK_MAX_VPT) {
    uint32_t w0 = 0, w1 = 0, w2 = 0, w3 = 0;
#pragma unroll
    for (int j = 0; j < EPV; ++j) {
      if (j < tail) {
        uint32_t bits;
        if (DT == DDTREE_BF16) bits = ((const uint16_t*)(base + (size_t)nvec_full * 16))[j];
        else bits = ((const uint32_t*)(base + (size_t)nvec_full * 16))[j];
        const int word = (DT == DDTREE_BF16) ? (j >> 1) : j;
        const uint32_t val = (DT == DDTREE_BF16) ? (bits << (16 * (j & 1))) : bits;
        if (word == 0) w0 |= val;
        else if (word == 1) w1 |= val;
        else if (word == 2) w2 |= val;
        else w3 |= val;
      }
    }
    const int vt = nvec_full / TOPK_THREADS;
#pragma unroll
    for (int v = 0; v < TOPK_MAX_VPT; ++v)
      if (v == vt) vec[v] = make_uint4(w0, w1, w2, w3);
  }

  // ---- keys, NaN check, chunk maximum ----
  auto raw_at = [&](int e) -> uint32_t {   // e-th element of this thread (bits)
    const int v = e / EPV, j = e % EPV;
    if (DT == DDTREE_BF16) return (u32_at(vec[v], j >> 1) >> (16 * (j & 1))) & 0xFFFFu;
    return u32_at(vec[v], j);
  };
  auto lid_at = [&](int e) -> int { return ((e / EPV) * TOPK_THREADS + tid) * EPV + (e % EPV); };
  auto lkey_at = [&](int e) -> LKey {
    const int lid = lid_at(e);
    if (lid >= len) return 0;
    uint32_t bits = raw_at(e);
    LKey k = (DT == DDTREE_BF16) ? (LKey)key16_of_bf16((uint16_t)bits) : (LKey)key32_of_f32(__uint_as_float(bits));
    return (k << LID_BITS) | (LKey)(LID_MASK - (uint32_t)lid);
  };

  LKey kmax_t = 0;
  bool nan_seen = false;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (lid_at(e) < len) {
      uint32_t bits = raw_at(e);
      nan_seen |= (DT == DDTREE_BF16) ? bf16_is_nan((uint16_t)bits) : (__uint_as_float(bits) != __uint_as_float(bits));
      LKey k = lkey_at(e);
      kmax_t = k > kmax_t ? k : kmax_t;
    }
  }
  if (__any_sync(0xffffffffu, nan_seen) && (tid & 31) == 0) flag_status(DDTREE_STATUS_NONFINITE);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    LKey w = __shfl_xor_sync(0xffffffffu, kmax_t, o);
    kmax_t = w > kmax_t ? w : kmax_t;
  }
  if ((tid & 31) == 0) red_k[tid >> 5] = kmax_t;
  __syncthreads();
  LKey kmax = red_k[0];
  for (int i = 1; i < TOPK_THREADS / 32; ++i) kmax = red_k[i] > kmax ? red_k[i] : kmax;
  const uint32_t vkey_max = (uint32_t)(kmax >> LID_BITS);
  const float m = (DT == DDTREE_BF16) ? bf16_of_key16(vkey_max) : f32_of_key32(vkey_max);

  // ---- sum of exp(z - m); for bf16 also the max-anchored window histogram ----
  for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0;
  __syncthreads();
  double s = 0.0;
  const bool m_finite = m > -INFINITY;
  const double md = (double)m;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (lid_at(e) < len) {
      uint32_t bits = raw_at(e);
      float z = (DT == DDTREE_BF16) ? bf16_bits_to_f32((uint16_t)bits) : __uint_as_float(bits);
      if (m_finite) s += exp((double)z - md);
      if (DT == DDTREE_BF16) {
        uint32_t d = vkey_max - key16_of_bf16((uint16_t)bits);
        if (d < 256u) atomicAdd(&hist[d], 1u);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((tid & 31) == 0) red_d[tid >> 5] = s;
  __syncthreads();

  // ---- local threshold ----
  LKey thr;
  {
    auto each = [&](auto f) {
#pragma unroll
      for (int e = 0; e < E; ++e) f(lkey_at(e));
    };
    int shift_done = T::KEY_BITS + LID_BITS;
    LKey prefix = 0;
    int need = kloc;
    bool have = false;
    if (DT == DDTREE_BF16) {
      // warp 0 scans the window: bin b holds the value vkey_max - b
      if (tid < 32) {
        uint32_t cbin[8];
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { cbin[j] = hist[8 * tid + j]; mine += cbin[j]; }
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += v;
        }
        uint32_t before = incl - mine;     // count in bins < 8*tid (closer to the max)
        bool here = before < (uint32_t)need && (uint32_t)need <= incl;
        unsigned msk = __ballot_sync(0xffffffffu, here);
        if (tid == 0) bcast[3] = msk ? 1 : 0;
        if (msk && tid == __ffs(msk) - 1) {
          uint32_t acc = before;
          int j = 0;
          for (; j < 7; ++j) {
            if (acc + cbin[j] >= (uint32_t)need) break;
            acc += cbin[j];
          }
          bcast[0] = 8 * tid + j;
          bcast[1] = need - (int)acc;
          bcast[2] = (int)cbin[j];
        }
      }
      __syncthreads();
      if (bcast[3]) {
        const uint32_t tval = vkey_max - (uint32_t)bcast[0];
        prefix = ((LKey)tval) << LID_BITS;
        need = bcast[1];
        shift_done = LID_BITS;
        have = (bcast[2] == need);
      }
      __syncthreads();
    }
    thr = have ? prefix : radix_select<LKey>(each, shift_done, prefix, need, hist, bcast);
  }

  // ---- emit the local candidates and the chunk statistics ----
  if (tid == 0) s_count = 0;
  __syncthreads();
  unsigned long long* cand_row = ws.cand + (size_t)row * plan.cand;
  unsigned long long* cand = cand_row + (size_t)c * plan.kmax;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    LKey k = lkey_at(e);
    if (k != 0 && k >= thr) {
      int slot = atomicAdd(&s_count, 1);
      const uint32_t vkey = (uint32_t)(k >> LID_BITS);
      const uint32_t gid = (uint32_t)(c0 + (LID_MASK - (uint32_t)(k & LID_MASK)));
      if (slot < kloc)
        cand[slot] = ((unsigned long long)vkey << TOPK_ID_BITS) | (unsigned long long)(TOPK_ID_MASK - gid);
    }
  }
  if (tid == 0) {
    double tot = 0.0;
    for (int i = 0; i < TOPK_THREADS / 32; ++i) tot += red_d[i];
    ws.stats[(size_t)row * plan.cpr + c] = make_double2(md, tot);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    unsigned t = atomicAdd(&ws.ticket[row], 1u);
    s_last = (t == (unsigned)(plan.cpr - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // =================== merge (last CTA of this row) ===================
  unsigned long long* sc = (unsigned long long*)smem_raw;           // [plan.cand]
  int kpow = 1;
  while (kpow < K) kpow <<= 1;
  unsigned long long* win = sc + plan.cand;                         // [kpow]
  const int ncand = plan.cand;
  for (int i = tid; i < ncand; i += TOPK_THREADS) sc[i] = __ldcg(cand_row + i);
  for (int i = tid; i < kpow; i += TOPK_THREADS) win[i] = 0ull;
  if (tid == 0) s_count = 0;
  __shared__ double s_lse;
  if (tid == 0) {
    double M = -INFINITY;
    for (int i = 0; i < plan.cpr; ++i) M = fmax(M, __ldcg(&ws.stats[(size_t)row * plan.cpr + i].x));
    double S = 0.0;
    if (M > -INFINITY) {
      for (int i = 0; i < plan.cpr; ++i) {
        double2 st = __ldcg(&ws.stats[(size_t)row * plan.cpr + i]);
        if (st.x > -INFINITY) S += st.y * exp(st.x - M);
      }
    }
    s_lse = M + log(S);
    ws.ticket[row] = 0;   // leave the workspace ready for the next call
  }
  __syncthreads();

  const int per = (ncand + TOPK_THREADS - 1) / TOPK_THREADS;
  auto gget = [&](int i) -> unsigned long long {
    int idx = i * TOPK_THREADS + tid;
    return idx < ncand ? sc[idx] : 0ull;
  };
  const int gbits = T::KEY_BITS + TOPK_ID_BITS;
  auto geach = [&](auto f) {
    for (int i = 0; i < per; ++i) f(gget(i));
  };
  unsigned long long gthr = radix_select<unsigned long long>(geach, gbits, 0ull, K, hist, bcast);
  for (int i = 0; i < per; ++i) {
    unsigned long long k = gget(i);
    if (k != 0 && k >= gthr) {
      int slot = atomicAdd(&s_count, 1);
      if (slot < kpow) win[slot] = k;
    }
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= kpow; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < kpow / 2; i += TOPK_THREADS) {
        int lo = 2 * stride * (i / stride) + (i % stride);
        int hi = lo + stride;
        bool desc = ((lo & size) == 0);
        unsigned long long a = win[lo], b = win[hi];
        if ((a < b) == desc) { win[lo] = b; win[hi] = a; }
      }
      __syncthreads();
    }
  }
  const double lse = s_lse;
  for (int i = tid; i < K; i += TOPK_THREADS) {
    unsigned long long k = win[i];
    uint32_t vkey = (uint32_t)(k >> TOPK_ID_BITS);
    int id = (int)(TOPK_ID_MASK - (uint32_t)(k & TOPK_ID_MASK));
    float z = (DT == DDTREE_BF16) ? bf16_of_key16(vkey) : f32_of_key32(vkey);
    out_ids[(size_t)row * K + i] = id;
    out_lp[(size_t)row * K + i] = (float)((double)z - lse);   // one rounding of the fp64 value
  }
  if (out_lse != nullptr && tid == 0) out_lse[row] = (float)lse;
}

inline size_t topk_smem_bytes(const TopkPlan& p, int K) {
  int kpow = 1;
  while (kpow < K) kpow <<= 1;
  return (size_t)(p.cand + kpow) * 8;
}

}  // namespace ddt
