// Verify-layer neighbour: the target's LM head with its argmax in the GEMM
// epilogue, so the [rows x V] logits are never written.
//
// "DDTree Deep Dive" §6: the verifier needs only the target's token at every
// tree node (its argmax at temperature 0).  With the logits computed here,
// tile by tile in tensor memory, the accept stage's pass over n x V logits
// in HBM (20 MB at B = 64, 78 MB at B = 256) disappears; what remains is one
// read of the LM-head weight and of the nodes' hidden states.
//
// logits[row][v] = sum_k hidden[row][k] * weight[v][k]  (bf16 x bf16 -> fp32)
// out[row] = the lowest v among the maxima of logits[row][0..V).
//
// Tiles: M = 128 rows (hidden), N = 256 vocabulary entries (weight rows),
// K steps of 64 (one 128-byte swizzle atom of each operand), both operands
// K-major in shared memory, loaded by TMA (no multicast), accumulated by
// tcgen05.mma (kind::f16) in tensor memory.  Persistent CTAs walk the tiles
// N-major (tile t = n * MT + m), so the CTAs of one wave share the weight
// tile through L2 and the weight is read from HBM once.
// Warps (192 threads): 0 TMA producer, 1 TMEM allocation and MMA issuer,
// 2-5 epilogue (warp w reads TMEM lanes 32 (w % 4) ..: one row per thread).
// Two accumulators of 256 columns alternate between tiles, so the epilogue
// of one tile overlaps the products of the next.  The epilogue reduces its
// row's 256 logits to (max, lowest index) and merges it into the row's
// 64-bit slot (order key of the fp32 maximum, complemented index) with
// atomicMax; the CTA that finishes the last tile (a ticket; nobody waits)
// publishes every row's argmax and resets the slots.  Every mbarrier wait is
// bounded as in the attention kernels.
#pragma once

#include "attn_tc.cuh"
#include "topk.cuh"

namespace ddt {

constexpr int LM_THREADS = 192;
constexpr int LM_BM = 128;
constexpr int LM_BN = 256;
constexpr int LM_BK = 64;
constexpr int LM_STAGES = 4;
constexpr int LM_A_TILE = LM_BM * LM_BK * 2;   // 16 KB
constexpr int LM_B_TILE = LM_BN * LM_BK * 2;   // 32 KB
constexpr uint32_t LM_TMEM_COLS = 512;

struct LmSmem {
  unsigned char a[LM_STAGES][LM_A_TILE];
  unsigned char b[LM_STAGES][LM_B_TILE];
  uint64_t full[LM_STAGES], empty[LM_STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
  int last;
};

constexpr size_t lm_smem_bytes() { return sizeof(LmSmem); }

struct LmWs {
  unsigned long long* slot;   // [rows] (order key << 20 | complemented index), 0 = none
  uint32_t* ticket;           // [1] finished tiles
};

inline size_t lm_ws_bytes(int rows) { return align256((size_t)rows * 8) + 256; }
inline LmWs lm_ws_carve(void* ws, int rows) {
  LmWs w;
  w.slot = (unsigned long long*)ws;
  w.ticket = (uint32_t*)((char*)ws + align256((size_t)rows * 8));
  return w;
}

struct LmParams {
  int rows, V, d;
  int mt, nt;                 // M-tiles, N-tiles
  int32_t* out;               // [rows]
  float* out_max;             // [rows] or null
  LmWs ws;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(LM_THREADS, 1)
lmhead_argmax_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                     const LmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  LmSmem& sm = *reinterpret_cast<LmSmem*>(smem_dyn);
  if ((smem_u32(smem_dyn) & 1023u) != 0u) {
    if (threadIdx.x == 0) flag_status(DDTREE_STATUS_SETUP);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles = p.mt * p.nt;
  const int ksteps = p.d / LM_BK;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles = tiles > (int)blockIdx.x ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  if (tid == 0) {
    for (int s = 0; s < LM_STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 128);
    }
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                 "r"(LM_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  const uint64_t wlim = p.wait_ns;

  if (warp == 0) {
    // =========================== TMA producer ===========================
    if (lane == 0) {
      int it = 0, issued = 0;
      bool ok = true;
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        const int m = t % p.mt, n = t / p.mt;
        for (int k = 0; k < ksteps; ++k, ++it) {
          const int s = it % LM_STAGES, use = it / LM_STAGES;
          if (use > 0 && !mbar_wait(&sm.empty[s], (use - 1) & 1, abort, wlim)) { ok = false; break; }
          mbar_expect_tx(&sm.full[s], LM_A_TILE + LM_B_TILE);
          tma_load_4d(smem_u32(sm.a[s]), &tm_h, &sm.full[s], k * LM_BK, m * LM_BM, 0, 0);
          tma_load_4d(smem_u32(sm.b[s]), &tm_w, &sm.full[s], k * LM_BK, n * LM_BN, 0, 0);
          issued = it + 1;
        }
      }
      if (*abort) {           // copies in flight must land before the CTA exits
        int z = 0;
        for (int j = max(0, issued - LM_STAGES); j < issued; ++j)
          mbar_wait(&sm.full[j % LM_STAGES], (j / LM_STAGES) & 1, (volatile int*)&z);
      }
    }
  } else if (warp == 1) {
    // =========================== MMA issuer ===========================
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(LM_BM, LM_BN, false, false);
      int it = 0;
      bool ok = true, any = false;
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int b = i & 1;
        if (i >= 2 && !mbar_wait(&sm.acc_empty[b], ((i >> 1) - 1) & 1, abort, wlim)) break;
        tc_fence_after();
        const uint32_t acc = tmem + LM_BN * b;
        for (int k = 0; k < ksteps; ++k, ++it) {
          const int s = it % LM_STAGES;
          if (!mbar_wait(&sm.full[s], (it / LM_STAGES) & 1, abort, wlim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm.a[s]), b_addr = smem_u32(sm.b[s]);
#pragma unroll
          for (int kk = 0; kk < LM_BK / 16; ++kk)
            umma_f16(acc, smem_desc_sw128(a_addr + kk * 32, 16, 1024), smem_desc_sw128(b_addr + kk * 32, 16, 1024),
                     IDESC, (k > 0 || kk > 0));
          umma_commit(&sm.empty[s]);
          any = true;
        }
        if (!ok) break;
        umma_commit(&sm.acc_full[b]);
      }
      if (*abort && any) {   // products in flight retire before the tensor memory is freed
        int z = 0;
        const int last = it - 1;
        mbar_wait(&sm.empty[last % LM_STAGES], (last / LM_STAGES) & 1, (volatile int*)&z);
      }
    }
  } else {
    // =========================== epilogue ===========================
    const int row_in_tile = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      const int t = (int)blockIdx.x + i * (int)gridDim.x;
      const int m = t % p.mt, n = t / p.mt;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[b], (i >> 1) & 1, abort, wlim))) break;
      tc_fence_after();
      const int v0 = n * LM_BN;
      float best = -INFINITY;
      int bidx = -1;
#pragma unroll 1
      for (int c = 0; c < LM_BN / 32; ++c) {
        float x[32];
        tmem_ld32(tmem + LM_BN * b + lane_off + c * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int v = v0 + c * 32 + e;
          if (v < p.V && (x[e] > best || (bidx < 0 && x[e] == best))) { best = x[e]; bidx = v; }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[b]);          // the accumulator is free for tile i + 2
      const int row = m * LM_BM + row_in_tile;
      if (row < p.rows && bidx >= 0)
        atomicMax(&p.ws.slot[row], ((unsigned long long)key32_of_f32(best) << TOPK_ID_BITS) |
                                       (unsigned long long)(TOPK_ID_MASK - (uint32_t)bidx));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(LM_TMEM_COLS));
  }
  // the CTA that finishes last publishes every row and resets the slots
  __threadfence();
  __syncthreads();
  if (tid == 0)
    sm.last = (my_tiles > 0 &&
               atomicAdd(p.ws.ticket, (uint32_t)my_tiles) + (uint32_t)my_tiles == (uint32_t)tiles) ? 1 : 0;
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  for (int r = tid; r < p.rows; r += LM_THREADS) {
    const unsigned long long s = __ldcg(&p.ws.slot[r]);
    p.ws.slot[r] = 0ull;
    p.out[r] = s == 0ull ? -1 : (int32_t)(TOPK_ID_MASK - (uint32_t)(s & TOPK_ID_MASK));
    if (p.out_max) p.out_max[r] = s == 0ull ? -INFINITY : f32_of_key32((uint32_t)(s >> TOPK_ID_BITS));
  }
  if (tid == 0) *p.ws.ticket = 0u;
}

// 2-D bf16 map over (K, rows) with a (64, box_rows) box and 128B swizzle.
inline bool make_map_2d_k(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {K, rows, 1, 1};
  cuuint64_t strides[3] = {K * 2, K * 2 * rows, K * 2 * rows};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult res = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

inline int lmhead_launch(const void* hidden, const void* weight, int rows, int V, int d, int32_t* out,
                         float* out_max, void* ws, int num_sms, cudaStream_t stream, uint64_t wait_ns) {
  LmParams p;
  p.rows = rows;
  p.V = V;
  p.d = d;
  p.mt = (rows + LM_BM - 1) / LM_BM;
  p.nt = (V + LM_BN - 1) / LM_BN;
  p.out = out;
  p.out_max = out_max;
  p.ws = lm_ws_carve(ws, rows);
  p.wait_ns = wait_ns > 0 ? wait_ns : TC_WAIT_NS;
  CUtensorMap mh, mw;
  if (!make_map_2d_k(&mh, hidden, (uint64_t)d, (uint64_t)rows, LM_BM) ||
      !make_map_2d_k(&mw, weight, (uint64_t)d, (uint64_t)V, LM_BN))
    return cuda_fail_msg("LM-head argmax: tensor maps");
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(lmhead_argmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lm_smem_bytes());
    if (e != cudaSuccess) return cuda_fail(e, "LM-head argmax: shared-memory attribute");
    attr_set = true;
  }
  const long long tiles = (long long)p.mt * p.nt;
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  lmhead_argmax_kernel<<<grid, LM_THREADS, lm_smem_bytes(), stream>>>(mh, mw, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "LM-head argmax: launch");
  return DDTREE_OK;
}

}  // namespace ddt
