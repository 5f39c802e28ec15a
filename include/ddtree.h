/*
 * ddtree.h - C ABI of the DDTree round library (libddtree.so), sm_100a.
 *
 * One DDTree draft-and-verify round, as described in "DDTree Deep Dive:
 * Algorithm, Code, and Engineering Philosophy of Block Diffusion Draft
 * Trees" (zhichai.net; below "Deep Dive") and "DDTree: Turning Block
 * Diffusion Drafters into Tree-Based Speculative Decoders" (alanhou.org):
 *
 *   ddtree_topk       per-position log-softmax and top-K of the drafter's
 *                     block logits                    (Deep Dive §1, §2 Lemma 1)
 *   ddtree_build      best-first heap over rank tuples -> prefix-closed tree
 *                     with parents, depths and ancestor bitmasks
 *                                                     (Deep Dive §2 Props. 2-3, §3)
 *   ddtree_tree_attn  ancestor-only attention of the B+1 tree nodes over
 *                     the committed KV prefix         (Deep Dive §4)
 *   ddtree_accept     greedy verifier walk + in-place KV compaction
 *                                                     (Deep Dive §5, §6)
 *   ddtree_round      the four stages in stream order, no host sync
 *
 * Conventions (all entry points):
 *  - Every pointer argument named as device memory must point to memory of
 *    the current CUDA device.  The caller owns every buffer; the library
 *    allocates nothing.  Scratch memory is the caller's workspace `ws` of at
 *    least the matching *_workspace_bytes(); it must be zero-filled once
 *    before its first use, and every call leaves its counters at zero again.
 *    Distinct calls that run concurrently need distinct workspaces.
 *  - Device pointers must be 16-byte aligned; logits rows must start on
 *    16-byte boundaries (row_stride * element size a multiple of 16).
 *  - Every call is asynchronous on `stream`.  The return value reports
 *    argument and launch errors synchronously (ddtree_status).  Data errors
 *    found on the device (NaN logits, a prefix that does not fit the cache)
 *    are OR-ed into a device status word that ddtree_device_status() reads.
 *  - Integer outputs are bit-exact functions of the inputs.  Ties are broken
 *    by lower token id (top-K, argmax) and lower rank tuple (tree order).
 *  - Limits: 1 <= L <= 32, 1 <= K <= min(V, 1024), 0 <= B <= 1024,
 *    1 <= n_req <= 4096, V <= 1048576, D in {64, 128}, Hq % Hkv == 0,
 *    page size 64.
 */
#ifndef DDTREE_H
#define DDTREE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DDTREE_OK = 0,
  DDTREE_ERR_INVALID_ARG = 1,  /* bad size, null or misaligned pointer */
  DDTREE_ERR_UNSUPPORTED = 2,  /* valid request outside what is built */
  DDTREE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  DDTREE_ERR_NONFINITE = 4,    /* device status bit: NaN in logits */
  DDTREE_ERR_TIMEOUT = 5,      /* device status bit: a bounded wait gave up */
  DDTREE_ERR_CAPACITY = 6,     /* device status bit: prefix + tree exceeds the cache */
  DDTREE_ERR_SCRATCH_LIMIT = 7 /* request needs more than the built-in scratch of ddtree_topk_static_ws */
} ddtree_status;

/* Device status word bits (ddtree_device_status). */
#define DDTREE_STATUS_NONFINITE 0x1u
#define DDTREE_STATUS_TIMEOUT   0x2u
#define DDTREE_STATUS_CAPACITY  0x4u
#define DDTREE_STATUS_SETUP     0x8u   /* a kernel could not set up (misaligned shared memory) and did nothing */
#define DDTREE_STATUS_BOUNDS    0x10u  /* debug build (DDTREE_DEBUG) only: an internal index left its range;
                                          the access was skipped */

typedef enum { DDTREE_BF16 = 0, DDTREE_F32 = 1 } ddtree_dtype;

#define DDTREE_PAGE 64

/*
 * KV cache geometry (Deep Dive §5: tree K/V sit in the cache tail).
 * Request r's committed prefix occupies logical slots 0..P_r-1 and its tree
 * node j occupies slot P_r + j.
 *   paged == 0: k/v are contiguous [layers][n_req][s_max][Hkv][D].
 *   paged == 1: k/v are pools [layers][num_blocks][64][Hkv][D]; logical slot
 *               s of request r is row s % 64 of block block_table[r][s / 64];
 *               block_table is int32 [n_req][max_blocks] in device memory.
 * Element type is the call's dtype.
 */
typedef struct {
  int layers;
  int n_req;
  int Hq;
  int Hkv;
  int D;
  float scale;       /* softmax scale; <= 0 selects 1/sqrt(D) */
  int paged;
  int s_max;         /* contiguous: slots per request */
  int num_blocks;    /* paged: pool blocks per layer */
  int max_blocks;    /* paged: block_table row length (logical capacity 64*max_blocks) */
} ddtree_kv_desc;

/* ---------------------------------------------------------------------- */
/* Stage 1: top-K + log-softmax (Deep Dive §1 and §2 Lemma 1).            */
/* ---------------------------------------------------------------------- */

size_t ddtree_topk_workspace_bytes(int rows, int V, int K);

/*
 * logits     device, [rows][row_stride] of dtype; only the first V entries
 *            of a row are read (rows = n_req * L block positions).
 * K          tokens kept per row, 1 <= K <= min(V, 1024).
 * ids        device int32 [rows][K]: token ids by (logit desc, id asc).
 * lp         device float [rows][K]: log q of those tokens, z - lse.
 * lse        device float [rows] (may be NULL): max + log S.
 * NaN logits set DDTREE_STATUS_NONFINITE; -inf is allowed and ranks last;
 * -0.0 ranks equal to +0.0.
 * lp is the fp64 value z - lse rounded once to fp32 (the sum of exp is taken
 * in fp64).  The first bf16 call on a device builds a 512 KiB table of
 * exp(z) for every bf16 value in static device memory and synchronizes
 * `stream` once; make it before any stream capture.
 */
int ddtree_topk(const void* logits, int dtype, int rows, int V, long long row_stride,
                int K, int32_t* ids, float* lp, float* lse,
                void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Stage 2: tree build (Deep Dive §2 Propositions 2 and 3, §3, §4).       */
/* ---------------------------------------------------------------------- */

/*
 * ids, lp    device [n_req][L][K] as written by ddtree_topk (lp sorted
 *            non-increasing within a row).
 * root_token device int32 [n_req]: the bonus token b of each request.
 * B          node budget: non-root nodes, 0 <= B <= 1024.
 * Outputs, n = B + 1 rows per request, node 0 = root, nodes 1.. in pop
 * order (so parent[i] < i); rows at or past n_nodes[r] are filled with
 * token/parent/depth/rank -1, score -inf and an all-zero mask:
 *   node_token int32 [n_req][n]   token of the node (root: root_token)
 *   parent     int32 [n_req][n]   parent node (root: -1)
 *   depth      int32 [n_req][n]   block position of the node (root: 0)
 *   node_rank  int32 [n_req][n]   rank of the token within its position's top-K
 *   score      float [n_req][n]   fp32 sum of lp along the path, one add per
 *                                 depth in root-to-leaf order (root: 0)
 *   anc        uint32 [n_req][n][W], W = ceil(n/32): bit j of row i (word
 *              j/32, bit j%32) is set iff node j is i or an ancestor of i
 *   n_nodes    int32 [n_req]: 1 + number of popped prefixes
 * The popped set is the top-B of all prefixes of length <= L under the order
 * (score desc, rank tuple lexicographically asc).  Any output pointer other
 * than parent, anc and n_nodes may be NULL.
 */
int ddtree_build(const int32_t* ids, const float* lp, const int32_t* root_token,
                 int n_req, int L, int K, int B,
                 int32_t* node_token, int32_t* parent, int32_t* depth,
                 int32_t* node_rank, float* score, uint32_t* anc, int32_t* n_nodes,
                 cudaStream_t stream);

/*
 * ddtree_build_ex: ddtree_build with two options and a diagnostic output.
 *
 * gain_floor device float [n_req] or NULL.  Adaptive budget ("DDTree Deep
 *            Dive" §10, cost-aware budgets; the autobench page's note that
 *            a bigger tree is not faster: the budget has an optimum).  Each
 *            pop adds its surrogate gain q(u) = exp(score) to the expected
 *            accepted length (Proposition 1), and pops come in non-increasing
 *            score order, so the tree that maximises sum q(u) - c*|T| among
 *            trees of at most B nodes is the leading run of pops with
 *            q(u) > c.  Request r keeps exactly the pops whose fp32 score is
 *            strictly greater than gain_floor[r] = log(c_r) (c_r: the
 *            verification cost of one more node, in accepted tokens); a NaN
 *            floor keeps no node.  n_nodes[r] = 1 + the kept pops, and rows
 *            past it are filled as for an exhausted tree.  NULL: no floor.
 * flags      0, or DDTREE_BUILD_FORCE_HEAP: select by Proposition 3's heap
 *            even when the threshold enumeration applies (same result;
 *            diagnostics and tests).
 * build_path device int32 [n_req] or NULL: which selection ran for the
 *            request: DDTREE_BUILD_PATH_ENUM (threshold enumeration, or
 *            B == 0), _HEAP_REG3 / _HEAP_REG9 (register-resident heap for
 *            B+1 <= 96 / 288), _HEAP_TOURNAMENT (block tournament heap).
 *            The enumeration falls back to the heap when more than 4096
 *            prefixes reach its score threshold.
 */
#define DDTREE_BUILD_FORCE_HEAP 0x1
#define DDTREE_BUILD_PATH_ENUM 0
#define DDTREE_BUILD_PATH_HEAP_REG3 1
#define DDTREE_BUILD_PATH_HEAP_REG9 2
#define DDTREE_BUILD_PATH_HEAP_TOURNAMENT 3
int ddtree_build_ex(const int32_t* ids, const float* lp, const int32_t* root_token,
                    int n_req, int L, int K, int B,
                    int32_t* node_token, int32_t* parent, int32_t* depth,
                    int32_t* node_rank, float* score, uint32_t* anc, int32_t* n_nodes,
                    const float* gain_floor, int flags, int32_t* build_path,
                    cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Stage 3: ancestor-only tree attention (Deep Dive §4).                  */
/* ---------------------------------------------------------------------- */

/*
 * ddtree_tree_kv_write: the verify layer's neighbour before tree attention
 * ("DDTree Deep Dive" §3, tree_compile: a node's position id is P + depth,
 * siblings share it; §5: node i's K/V sit at cache slot P + i).  For every
 * layer, request r and live node i < n_nodes[r]:
 *   q_out[l][r][i] = rope(q_in[l][r][i], P_r + depth[r][i])   (if q_in)
 *   K cache slot P_r + i = rope(k_in[l][r][i], P_r + depth[r][i])
 *   V cache slot P_r + i = v_in[l][r][i]
 * rope: the rotary position embedding (Su et al., "RoFormer", §3.4) with the
 * half-split pairing: for i < D/2 the pair (x_i, x_{i+D/2}) turns by the
 * angle pos * rope_theta^(-2i/D) (the Qwen3 family uses rope_theta = 1e6);
 * rope_theta <= 0 writes K unrotated.  The angles are computed in fp64, the
 * rotation in fp32, the result rounded to the dtype.
 * q_in, q_out  device [layers][n_req][B+1][Hq][D] or both NULL; q_out may
 *              alias q_in.
 * k_in, v_in   device [layers][n_req][B+1][Hkv][D].
 * depth, n_nodes  device, from ddtree_build.  prefix_len device [n_req].
 * A request whose tree does not fit its cache (or whose block-table entry is
 * out of range) is skipped and flags DDTREE_STATUS_CAPACITY.
 */
int ddtree_tree_kv_write(const void* q_in, void* q_out, const void* k_in, const void* v_in, int dtype,
                         const int32_t* depth, const int32_t* n_nodes, const int32_t* prefix_len,
                         const ddtree_kv_desc* kv, const int32_t* block_table, int B, double rope_theta,
                         void* k_cache, void* v_cache, cudaStream_t stream);

size_t ddtree_attn_workspace_bytes(const ddtree_kv_desc* kv, int B);

/*
 * q          device [layers][n_req][B+1][Hq][D] of dtype: tree-node queries
 *            (already rotated).
 * k_cache, v_cache  device, geometry `kv` (see ddtree_kv_desc).
 * prefix_len device int32 [n_req]: committed prefix P_r; P_r + n_nodes[r]
 *            must fit the request's capacity, else the request is skipped
 *            and DDTREE_STATUS_CAPACITY is set.
 * anc, n_nodes  device, as written by ddtree_build for budget B.
 * out        device [layers][n_req][B+1][Hq][D] of dtype: for node i < n_nodes
 *            and query head h (KV head h / (Hq/Hkv)), softmax(q k^T * scale) v
 *            over the prefix slots 0..P-1 and the tree slots P+j of every j set
 *            in anc[i].  Rows of absent nodes are not written.
 * out_lse    device float [layers][n_req][B+1][Hq] natural-log sum-exp of the
 *            scaled scores (may be NULL).
 * ws         device scratch of ddtree_attn_workspace_bytes(kv, B) bytes
 *            (16-byte aligned; NULL when that is 0).  It must be zero-filled
 *            before its first use; every call leaves its counters at zero.
 *            Calls that share a workspace must not overlap.
 * bf16 (D = 64 or 128): tcgen05 tensor-core kernels (fp32 accumulation, P
 * rounded to bf16 for the PV product); fp32: the CUDA-core fp32 kernel.
 */
int ddtree_tree_attn(const void* q, const void* k_cache, const void* v_cache, int dtype,
                     const ddtree_kv_desc* kv, const int32_t* block_table,
                     const int32_t* prefix_len, const uint32_t* anc, const int32_t* n_nodes,
                     int B, void* out, float* out_lse,
                     void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Stage 4: verifier walk + KV compaction (Deep Dive §5, §6).             */
/* ---------------------------------------------------------------------- */

size_t ddtree_accept_workspace_bytes(int n_req, int B, int V);

/*
 * target_logits device [n_req][B+1][row_stride] of dtype: the target's
 *            logits at every tree node (rows past n_nodes are not read).
 * node_token, parent, n_nodes  device, from ddtree_build.
 * prefix_len device int32 [n_req] (read only); new_prefix_len device int32
 *            [n_req] receives P + accept_len (must not alias prefix_len).
 * k_cache, v_cache, kv, block_table  the cache to compact in place; k_cache
 *            may be NULL to skip compaction.
 * Outputs per request (temperature 0):
 *   target_argmax int32 [n_req][B+1] (may be NULL): argmax of each live
 *                 node's row, lowest id on ties (-0.0 equals +0.0); NaN
 *                 entries are skipped (and flag DDTREE_STATUS_NONFINITE); a
 *                 row of NaN only gives -1, which matches no child
 *   path       int32 [n_req][L+1]: accepted node ids root first, -1 after
 *   accept_len int32 [n_req]: accepted draft nodes + 1 (the new bonus)
 *   next_bonus int32 [n_req]: target argmax at the last accepted node (-1
 *              when that node's row is NaN only)
 *   src_slot, dst_slot int32 [n_req][L+1]: P+path[j] -> P+j, -1 after
 * For every layer and both caches, slot P+path[j] is copied to slot P+j for
 * j = 0..accept_len-1; all sources are read before any destination is
 * written.  Any output pointer except new_prefix_len may be NULL.
 */
int ddtree_accept(const void* target_logits, int dtype, int V, long long row_stride,
                  const int32_t* node_token, const int32_t* parent, const int32_t* n_nodes,
                  int n_req, int L, int B,
                  const int32_t* prefix_len, int32_t* new_prefix_len,
                  void* k_cache, void* v_cache, const ddtree_kv_desc* kv,
                  const int32_t* block_table,
                  int32_t* target_argmax, int32_t* path, int32_t* accept_len,
                  int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot,
                  void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * ddtree_accept_ex: ddtree_accept at temperature > 0 ("DDTree Deep Dive" §6
 * and §9: tree verification that keeps the target distribution; the pages
 * give no rule, this is the plainest one that does).  With sampling NULL or
 * temperature <= 0 it is ddtree_accept.  Otherwise the target's token at
 * every live node is one draw from softmax(z / temperature) instead of the
 * argmax, and the walk is unchanged: each committed token is then a draw
 * from the target at its context.  The draw is the Gumbel-max identity,
 * argmax_v (z_v / T - log(-log u_v)), with
 *   u_v = ((w >> 12) + 1/2) * 2^-52,  w = word v % 4 of Philox4x64-10
 *         (Salmon et al., SC 2011) at counter (v / 4, node, request, 0)
 *         and key (seed, offset),
 * the score formed in fp64 (z times the fp64 value of 1/T, plus the
 * Gumbel term, each operation rounded) and rounded once to fp32; the
 * argmax takes the lowest id among equal fp32 scores.  target_argmax then
 * holds the drawn tokens.  Reuse (seed, offset) only to reproduce a round:
 * e.g. offset = the round index.  NaN or +inf temperature:
 * DDTREE_ERR_INVALID_ARG.
 */
typedef struct {
  double temperature;          /* > 0: draw; <= 0: greedy argmax */
  unsigned long long seed;     /* Philox key, first word */
  unsigned long long offset;   /* Philox key, second word */
} ddtree_sampling;

int ddtree_accept_ex(const void* target_logits, int dtype, int V, long long row_stride,
                     const int32_t* node_token, const int32_t* parent, const int32_t* n_nodes,
                     int n_req, int L, int B,
                     const int32_t* prefix_len, int32_t* new_prefix_len,
                     void* k_cache, void* v_cache, const ddtree_kv_desc* kv,
                     const int32_t* block_table,
                     int32_t* target_argmax, int32_t* path, int32_t* accept_len,
                     int32_t* next_bonus, int32_t* src_slot, int32_t* dst_slot,
                     const ddtree_sampling* sampling,
                     void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * The target's LM head with its argmax fused into the product ("DDTree Deep
 * Dive" §6: the verifier needs only the target's token at each node), so
 * the [rows][V] logits are never written:
 *   out_argmax[r] = lowest v maximising sum_k hidden[r][k] * weight[v][k]
 * with bf16 operands and fp32 accumulation on the tensor cores (the order of
 * that accumulation is the hardware's: two logits within its rounding of
 * each other may resolve either way).
 * hidden     device bf16 [rows][d] (e.g. the tree nodes' final hidden states,
 *            rows = n_req * (B+1)); weight device bf16 [V][d]; d % 64 == 0.
 * out_argmax device int32 [rows]; out_max device float [rows] (may be NULL):
 *            the maximum logit.
 * ws         device scratch of ddtree_lmhead_workspace_bytes(rows) bytes,
 *            zero-filled before first use; every call leaves it at zero.
 */
size_t ddtree_lmhead_workspace_bytes(int rows);
int ddtree_lmhead_argmax(const void* hidden, const void* weight, int rows, int V, int d,
                         int32_t* out_argmax, float* out_max, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/*
 * The verifier walk and KV compaction of ddtree_accept from given per-node
 * target tokens (target_token device int32 [n_req][B+1]: e.g. the output of
 * ddtree_lmhead_argmax, or drawn tokens).  Outputs, compaction and dtype
 * (of the caches) as for ddtree_accept.
 */
int ddtree_walk(const int32_t* target_token, const int32_t* node_token, const int32_t* parent,
                const int32_t* n_nodes, int n_req, int L, int B,
                const int32_t* prefix_len, int32_t* new_prefix_len,
                void* k_cache, void* v_cache, const ddtree_kv_desc* kv, const int32_t* block_table,
                int dtype, int32_t* path, int32_t* accept_len, int32_t* next_bonus,
                int32_t* src_slot, int32_t* dst_slot, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* The whole round (Deep Dive §3 stage pipeline: draft -> tree_build ->   */
/* tree_compile -> verify -> commit; the draft and the target forward are */
/* the caller's, their logits and Q/K/V are inputs here).                 */
/* ---------------------------------------------------------------------- */

typedef struct {
  /* sizes */
  int n_req, L, V, K, B;
  int dtype;                       /* of drafter logits, q, caches, target logits */
  ddtree_kv_desc kv;
  /* inputs (device) */
  const void* drafter_logits;      /* [n_req*L][drafter_stride] */
  long long drafter_stride;
  const int32_t* root_token;       /* [n_req] */
  const void* q;                   /* [layers][n_req][B+1][Hq][D] */
  void* k_cache;                   /* compacted in place */
  void* v_cache;
  const int32_t* block_table;      /* paged only */
  const int32_t* prefix_len;       /* [n_req] */
  const void* target_logits;       /* [n_req][B+1][target_stride] */
  long long target_stride;
  /* outputs (device) */
  int32_t* ids; float* lp; float* lse;                        /* stage 1 */
  int32_t* node_token; int32_t* parent; int32_t* depth;       /* stage 2 */
  int32_t* node_rank; float* score; uint32_t* anc; int32_t* n_nodes;
  void* attn_out; float* attn_lse;                            /* stage 3 */
  int32_t* target_argmax; int32_t* path; int32_t* accept_len; /* stage 4 */
  int32_t* next_bonus; int32_t* src_slot; int32_t* dst_slot;
  int32_t* new_prefix_len;
  /* scratch */
  void* ws; size_t ws_bytes;
  /* optional (NULL: none): per-request adaptive-budget floor of the build,
   * device float [n_req], as gain_floor of ddtree_build_ex */
  const float* gain_floor;
  /* optional (NULL: greedy): verification at temperature > 0, as for
   * ddtree_accept_ex */
  const ddtree_sampling* sampling;
  /* optional (tree_k_in NULL: none): the tree nodes' un-rotated Q, K, V
   * ([layers][n_req][B+1][H][D]); after the build the round runs
   * ddtree_tree_kv_write with them, writing the rotated Q into `q` (which
   * must then be writable; tree_q_in NULL leaves q as given) and K/V into the
   * cache tail, before the attention. */
  const void* tree_q_in;
  const void* tree_k_in;
  const void* tree_v_in;
  double rope_theta;
  /* optional (target_hidden NULL: none): the target's final hidden states of
   * the tree nodes, bf16 [n_req*(B+1)][d_model], and its LM head, bf16
   * [V][d_model]; the accept stage then takes each node's token from
   * ddtree_lmhead_argmax instead of target_logits (greedy only). */
  const void* target_hidden;
  const void* lm_head;
  int d_model;
  /* optional (NULL: none): 6 events the round records on `stream` at its
   * stage boundaries (before top-K, build, tree K/V write, attention and
   * accept, and after accept), for per-stage cudaEventElapsedTime; the round
   * also marks each stage with an NVTX range on the host. */
  cudaEvent_t* stage_events;
} ddtree_round_args;

/* Bytes of a->ws the round needs (0 for an invalid geometry).  The
 * workspace holds the stages' counters and tickets: it must be zero-filled
 * before its first use, and every call leaves them at zero again. */
size_t ddtree_round_workspace_bytes(const ddtree_round_args* a);

/* Stage order topk -> build -> tree_attn -> accept on `stream`; ids, lp,
 * node_token, parent, depth, anc, n_nodes and new_prefix_len are required,
 * the other outputs may be NULL. */
int ddtree_round(const ddtree_round_args* a, cudaStream_t stream);

/* Number of kernel launches one ddtree_round call with these arguments
 * makes on the current device (the one-time exp table build excluded), or
 * -1 for an invalid geometry.  Host only: no device work. */
int ddtree_round_launch_count(const ddtree_round_args* a);

/*
 * The round from host memory: the call a user makes whose drafter and
 * target produce their logits and tree-node Q/K/V on the host.  All copies
 * are cudaMemcpyAsync on `stream` (one per buffer, or one 2-D copy per
 * request for the tree K/V rows); use pinned host memory for them to
 * overlap.  In order on the stream:
 *   1. host -> device: drafter_logits, root_token, q, target_logits and
 *      prefix_len into the buffers of `dev` (same layouts); when tree_k and
 *      tree_v are given, the K and V rows of the B+1 tree nodes of every
 *      layer and request ([layers][n_req][B+1][Hkv][D] on the host) into
 *      cache slots P_r .. P_r + B (Deep Dive §5: tree K/V sit in the cache
 *      tail), P_r read from the host prefix_len;
 *   2. ddtree_round(dev);
 *   3. device -> host: every non-NULL output of `host` from the matching
 *      buffer of `dev`.
 * The call returns once everything is enqueued; synchronise `stream` before
 * reading the host outputs.  Host pointers left NULL are not copied (an
 * input then keeps whatever the device buffer holds).  Calls on different
 * streams with disjoint `dev` buffers and workspaces may run at the same
 * time: one round's copies then overlap another round's kernels.
 */
typedef struct {
  /* inputs (host) */
  const void* drafter_logits;      /* [n_req*L][drafter_stride] */
  const int32_t* root_token;       /* [n_req] */
  const void* q;                   /* [layers][n_req][B+1][Hq][D] */
  const void* target_logits;       /* [n_req][B+1][target_stride] */
  const int32_t* prefix_len;       /* [n_req] */
  const void* tree_k;              /* [layers][n_req][B+1][Hkv][D]; contiguous caches only */
  const void* tree_v;              /* (paged: DDTREE_ERR_UNSUPPORTED) */
  /* outputs (host) */
  void* attn_out;                  /* [layers][n_req][B+1][Hq][D] */
  int32_t* node_token;             /* [n_req][B+1] */
  int32_t* parent;                 /* [n_req][B+1] */
  int32_t* n_nodes;                /* [n_req] */
  int32_t* path;                   /* [n_req][L+1] */
  int32_t* accept_len;             /* [n_req] */
  int32_t* next_bonus;             /* [n_req] */
  int32_t* new_prefix_len;         /* [n_req] */
} ddtree_round_host_io;

int ddtree_round_host(const ddtree_round_args* dev, const ddtree_round_host_io* host, cudaStream_t stream);

/* Bytes ddtree_round_host copies host -> device (*h2d) and device -> host
 * (*d2h) with these arguments; -1 for invalid arguments.  Host only. */
int ddtree_round_host_bytes(const ddtree_round_args* dev, const ddtree_round_host_io* host,
                            unsigned long long* h2d, unsigned long long* d2h);

/* ---------------------------------------------------------------------- */
/* Top-K without a caller workspace (no counterpart in the paper: an      */
/* interface convenience of this library).                                */
/* ---------------------------------------------------------------------- */

/*
 * Same computation, arguments and results as ddtree_topk, but the scratch
 * memory lives in a fixed array built into the library instead of a
 * caller workspace, so the call allocates nothing and needs no workspace.
 * It is meant for callers that cannot allocate device memory while they
 * run rounds: serving engines that hand all free device memory to their KV
 * cache pool at start-up, where a cudaMalloc at decode time can synchronize
 * the device or fail because that pool already holds the memory.
 *
 * Limits and behaviour:
 *  - The built-in scratch is 4 MiB per device, held until the process
 *    exits.  A request whose scratch need for its own dtype exceeds it is
 *    rejected with DDTREE_ERR_SCRATCH_LIMIT before anything is launched (at
 *    V = 151936 and bf16 logits: up to 571 rows at K = 64, 145 at K = 256,
 *    48 at K = 1024 on a 148-SM B200).  ddtree_topk_workspace_bytes(rows,
 *    V, K) returns the larger of the bf16 and fp32 needs, so it bounds that
 *    need from above: a request it puts within 4 MiB is always accepted,
 *    but some it puts above 4 MiB are accepted too.
 *  - With CUDA's default lazy module loading, the device memory of the
 *    library's static arrays (this scratch and the 512 KiB exp table of
 *    ddtree_topk) is allocated when the library's module is first loaded on
 *    a device, which happens at the first call into it there.  Make one
 *    warm-up call per device at start-up, before the KV pool takes the free
 *    memory and before any stream capture: it performs that allocation,
 *    looks up the array's device address on the current device and, for
 *    bf16, builds the exp table (synchronizing `stream` once).  Later calls
 *    allocate nothing.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; each call clears the counters it needs at its start.  Calls
 *    that overlap on the GPU (other streams, other host threads) race on the
 *    array and must be serialized by the caller.
 */
int ddtree_topk_static_ws(const void* logits, int dtype, int rows, int V, long long row_stride, int K,
                          int32_t* ids, float* lp, float* lse, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Status                                                                 */
/* ---------------------------------------------------------------------- */

const char* ddtree_status_string(int status);

/* Synchronises `stream`, returns the device status word's bits in *bits and
 * clears it.  Returns DDTREE_OK or DDTREE_ERR_CUDA. */
int ddtree_device_status(cudaStream_t stream, unsigned int* bits);

/*
 * Diagnostics of the tensor-core attention kernel's timeout path (no
 * counterpart in the paper).  Every wait of that kernel's pipeline is
 * bounded; on timeout the kernel sets DDTREE_STATUS_TIMEOUT, every role
 * leaves its loop, waits (bounded by one second) for its own copies and
 * tensor-core products in flight, frees its tensor memory and returns, so
 * the context stays usable.  For tests of that path:
 *   wait_ns        limit of the pipeline's waits (0: the default, 1 s);
 *   withhold_tile  >= 0: the producer issues no key tile from this index
 *                  (within each CTA's key range) on, so a consumer's wait
 *                  runs out; -1: normal operation.
 * The setting is process-wide and applies to later ddtree_tree_attn and
 * ddtree_round calls until reset with (0, -1).  Outputs of a call that
 * timed out are undefined.  Returns DDTREE_ERR_INVALID_ARG for
 * withhold_tile < -1.
 */
int ddtree_debug_attn_timeout(unsigned long long wait_ns, int withhold_tile);

/*
 * Which attention kernel ddtree_tree_attn (and the round's attention stage)
 * launches for this cache geometry and tree budget B (no counterpart in the
 * paper; host-only, no device work).  dtype as in ddtree_tree_attn;
 * num_sms: the SM count to plan for (0: the current device's).  On
 * DDTREE_OK, *kernel is
 *   0  CUDA-core kernel (fp32, or a head grouping the tensor cores do not take),
 *   1  one M-tile of 128 rows per CTA (short key ranges),
 *   2  two M-tiles per CTA sharing each key tile (long key ranges; D = 64 always),
 * and *splits the number of key-range splits (1: no combine launch).
 * Returns DDTREE_ERR_INVALID_ARG / DDTREE_ERR_UNSUPPORTED as ddtree_tree_attn
 * would for the geometry, or for null outputs.
 */
int ddtree_attn_plan(const ddtree_kv_desc* kv, int B, int dtype, int num_sms, int* kernel, int* splits);

/* The call and the CUDA runtime's message behind the last DDTREE_ERR_CUDA
 * return of a host-side launch or set-up step (empty before any). */
const char* ddtree_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int ddtree_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DDTREE_H */
