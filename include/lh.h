/*
 * lh.h — C ABI of liblh, the sm_100a (B200) implementation of the Lighthouse
 * Attention hot path.
 *
 * Method: "Long Context Pre-Training with Lighthouse Attention" (Peng, Ghosh,
 * Quesnelle; arXiv 2605.06554), §3.1: a training-only wrapper around causal
 * scaled dot-product attention. Forward: (i) mean-pool Q, K and V into an
 * L-level pyramid with factor p; (ii) score pyramid entries by l2 norm and
 * select with a top-K descent; gather the selection, ordered by position,
 * into one causal sub-sequence; (iii) dense causal attention (Eq. (1)) on that
 * sub-sequence; (iv) scatter each output back onto the tokens its entry
 * covers. Backward (Fig. 1, gradient path): through the scatter, the
 * attention and the gather/pool; the selection takes no gradient.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to caller-owned, contiguous,
 *    16-byte aligned buffers. liblh never allocates device memory, never
 *    frees it, and never keeps a pointer after the call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). All work is enqueued asynchronously on it; no entry point
 *    synchronises the host except lh_get_device_error.
 *  - Arguments are validated before anything is launched; on any error
 *    nothing is launched and the status says why. LH_ERR_CUDA means a launch
 *    failed (cudaGetLastError was not cudaSuccess after it).
 *  - Element types: `dtype` buffers hold bf16 or fp32 per lh_config.dtype;
 *    buffers typed float / double / int32_t below are always that type.
 *  - liblh looks up the device address of its device error word (and, for
 *    lh_score_topk_noalloc, of its scratch array) once per device and keeps it
 *    for the life of the process. cudaDeviceReset unloads the library's device
 *    code and so invalidates those addresses: a process that resets a device
 *    must not call liblh on that device afterwards.
 *
 * Layouts (row-major, last index fastest):
 *   tokens  Q, K, V, O, dO, dQ, dK, dV     [B][N][H][D]   dtype
 *   pyramid pyr_q, pyr_k, pyr_v            [B][H][E][D]   dtype, levels 1..L-1
 *           (E = sum_{l>=1} n_l; level l starts at entry plan.lvl_off[l])
 *   squared norms sq                       [2][B][H][E]   double ([0]: query, [1]: key)
 *   selection sel                          [B][H][L-1][K] int32 (row l-1: level l)
 *   gather map                             [B][H][S]      int32, (level << 28) | index
 *   slot table                             [B][H][E]      int32, per entry of levels >= 1:
 *                                                         -1: not a candidate (pruned);
 *                                                         2*s: in the sub-sequence at slot s;
 *                                                         2*s + 1: expanded, and under
 *                                                         LH_INCL_NESTED in the sub-sequence
 *                                                         at slot s; under LH_INCL_PARTITION
 *                                                         not in it, s = the first slot of
 *                                                         its descendants' run
 *   sub-sequence qs, ks, vs, and dos       [B][H][S][D]   attention operand type: fp16 for
 *                                                         bf16 I/O (x * 2^-e, e the head's
 *                                                         exponent from `scale`), fp32 for
 *                                                         fp32 I/O
 *   operand scale                          [4][B][H]      uint32: the largest magnitude (fp32
 *                                                         bit pattern) of the head's queries,
 *                                                         keys, values (lh_pool) and dO block
 *                                                         sums (lh_scatter_bwd). The fp16
 *                                                         operands of bf16 I/O are x * 2^-e,
 *                                                         e = 0 while that magnitude is in
 *                                                         [4, 256), else the exponent that
 *                                                         brings it into [4, 8): a power of
 *                                                         two moves no significant bit, so
 *                                                         every bf16 value within 2^19 of its
 *                                                         head's largest enters exactly (bf16's
 *                                                         range beyond fp16's 65504 and below
 *                                                         its 2^-14 included), and the kernels
 *                                                         take the powers of two out of their
 *                                                         results. Magnitudes are handled from
 *                                                         2^-60 to 2^60.
 *   attention out os, grads dqs, dks, dvs  [B][H][S][D]   float
 *   lse, delta                             [B][H][S]      float
 */
#ifndef LH_H
#define LH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LH_MAX_LEVELS 8
#define LH_MAX_K 4096

typedef enum {
  LH_OK = 0,
  LH_ERR_NULL = 1,       /* a required pointer is NULL */
  LH_ERR_SHAPE = 2,      /* sizes outside the supported set (see lh_plan) */
  LH_ERR_ALIGN = 3,      /* a buffer is not 16-byte aligned */
  LH_ERR_DTYPE = 4,      /* unknown dtype */
  LH_ERR_MODE = 5,       /* unknown accumulation mode or reading (lh_score, lh_ties, lh_order, lh_weight,
                            lh_inclusion) */
  LH_ERR_WORKSPACE = 6,  /* workspace smaller than plan.ws_bytes */
  LH_ERR_CUDA = 7,       /* a CUDA launch or runtime call failed */
  LH_ERR_TIMEOUT = 8,    /* a bounded device-side wait gave up (reported by lh_get_device_error) */
  LH_ERR_DEVICE = 9      /* a device-side check failed (reported by lh_get_device_error) */
} lh_status;

typedef enum { LH_BF16 = 0, LH_FP32 = 1 } lh_dtype;

/* Accumulation of the steps that add several contributions into one token
 * (forward scatter, backward spread). The pages' scatter-back has an
 * fp-atomic default and a deterministic int-atomic variant ("Lighthouse
 * Attention Technique", throughput paragraph). Here each token's sum is
 * formed by the thread that owns the token (no atomics), so both modes are
 * run-to-run deterministic; they differ in arithmetic:
 *   LH_ACC_FP32    fp32 sum, coarse level first (counterpart of fp-atomic)
 *   LH_ACC_FIXED64 int64 fixed point, one count = 2^-32: each contribution
 *                  w*x is rounded to a count (x * 2^32 / p^l in double,
 *                  round half to even) and counts add exactly, so the result
 *                  is independent of summation order (counterpart of
 *                  int-atomic). Sums must stay below 2^31 in magnitude. */
typedef enum { LH_ACC_FP32 = 0, LH_ACC_FIXED64 = 1 } lh_accum;

/* Readings of points the pages leave open, selectable (value 0 = the reading
 * the library implements by default). The pages describe the score only as the
 * l2 norm of the pooled summaries, "bidirectional" over queries and keys
 * ("Long Context Pre-Training with Lighthouse Attention", §3.1 (ii) and Fig. 2);
 * the entry order only as sorted by position with causality kept (Fig. 1); the
 * scatter-back as distributing each output to the positions it represents
 * (§3.1 (iv)). Ranking uses squared norms where the order is the same. */
typedef enum {
  LH_SCORE_MAX = 0,    /* max(|mean_q|^2, |mean_k|^2) */
  LH_SCORE_K = 1,      /* |mean_k|^2 */
  LH_SCORE_SUM = 2,    /* |mean_q| + |mean_k| (fp64 square roots, then their sum) */
  LH_SCORE_PROD = 3,   /* |mean_q|^2 * |mean_k|^2 (same order as |mean_q| * |mean_k|) */
  LH_SCORE_MAXPOOL = 4 /* bottom-up: a token scores max(|q|^2, |k|^2), an entry the max of its
                          children's scores (lh_pool then writes tokens' norms max-pooled into sq) */
} lh_score;
typedef enum {
  LH_TIES_LOW_FIRST = 0,   /* equal scores: lower index first */
  LH_TIES_HIGH_FIRST = 1   /* equal scores: higher index first */
} lh_ties;
typedef enum {
  LH_ORDER_POST = 0,   /* by last covered token, finer level first (descendants before ancestors) */
  LH_ORDER_PRE = 1     /* by first covered token, coarser level first (ancestors before descendants) */
} lh_order;
typedef enum {
  LH_WEIGHT_ONE = 0,   /* forward scatter adds every covering entry's row with weight 1 */
  LH_WEIGHT_MEAN = 1   /* ... with weight 1/p^l (the block-sum backward takes the same weights) */
} lh_weight;
typedef enum {
  LH_INCL_NESTED = 0,    /* expanded entries stay in the sub-sequence (parents kept: Fig. 2) */
  LH_INCL_PARTITION = 1  /* expanded entries leave it: the included entries tile the tokens, each
                            token covered exactly once (the order readings then coincide) */
} lh_inclusion;

typedef struct {
  int B, H, N, D;   /* batch, heads, tokens, head dim (D in {64, 128}) */
  int p, L, K;      /* pool factor (>= 2), levels (1..LH_MAX_LEVELS), top-K budget (1..LH_MAX_K) */
  lh_dtype dtype;   /* element type of tokens, pyramid, sub-sequence, outputs */
  lh_accum accum;   /* accumulation mode of lh_scatter / lh_spread */
  lh_score score;   /* ranking score of pooled entries (lh_score_topk) */
  lh_ties ties;     /* tie-break of equal scores (lh_score_topk) */
  lh_order order;   /* entry order of the sub-sequence (lh_score_topk) */
  lh_weight weight; /* weights of the forward scatter and of its adjoint lh_scatter_bwd */
  lh_inclusion inclusion; /* whether expanded entries stay in the sub-sequence (lh_plan, lh_score_topk) */
} lh_config;

typedef struct {
  int S;                              /* sub-sequence length (same for every (b,h)) */
  int E;                              /* entries of levels 1..L-1 per (b,h) */
  int n[LH_MAX_LEVELS];               /* n_l = N / p^l */
  int k[LH_MAX_LEVELS];               /* entries expanded at level l (l >= 1) */
  int c[LH_MAX_LEVELS];               /* entries of level l in the sub-sequence */
  int lvl_off[LH_MAX_LEVELS];         /* start of level l (l >= 1) within E; lvl_off[0] = 0 unused */
  size_t ws_bytes;                    /* workspace bytes lh_score_topk / lh_forward need (0 if L == 1) */
} lh_plan_t;

/* Library version (major*10000 + minor*100 + patch). */
int lh_version(void);

/* Human-readable name of a status code (static string). */
const char* lh_status_string(lh_status s);

/* Sizes of one problem. Pure host function, no CUDA call.
 * Source: [LH] §1 size law S = O(LpK + N/p^(L-1)) under the descent reading:
 * candidates m_{L-1} = n_{L-1}; k_l = min(K, m_l); m_{l-1} = p * k_l; included
 * c_l = m_l (LH_INCL_NESTED) or m_l - k_l for l >= 1 (LH_INCL_PARTITION),
 * c_0 = m_0; S = sum of c_l. ws_bytes = 5 * (sum of m_l) int32 per (b,h).
 * Errors: LH_ERR_NULL, LH_ERR_SHAPE (B,H,N < 1; D not 64/128; p < 2;
 * L outside 1..LH_MAX_LEVELS; K outside 1..LH_MAX_K; N % p^(L-1) != 0;
 * N or the candidate total sum m_l >= 2^28), LH_ERR_DTYPE, LH_ERR_MODE. */
lh_status lh_plan(const lh_config* cfg, lh_plan_t* out);

/* (i) Pyramid pool + squared norms. [LH] §3.1 stage (i), Fig. 2 steps 1-2.
 * Also writes rows 0-2 (queries, keys, values) of `scale`: each head's largest
 * token magnitude (pooled means are no larger); for L = 1 only this is done.
 * For levels l = 1..L-1: entry i of pyr_x holds mean of tokens
 * [i p^l, (i+1) p^l), formed in fp64 level by level (each level's sum is the
 * left-to-right sum of its p children's sums) and rounded to nearest-even
 * into dtype. sq[0] / sq[1] hold the squared l2 norm of the fp64 query / key
 * means in a pinned order (8-component chunks summed left to right, chunk
 * partials combined by a stride-halving tree). Under LH_SCORE_MAXPOOL, sq[0] / sq[1]
 * hold instead the largest such squared norm among the entry's query / key
 * token rows. Nothing is written when L = 1.
 * Inputs q, k, v; outputs pyr_q, pyr_k, pyr_v, sq (may be NULL when L = 1), scale. */
lh_status lh_pool(const lh_config* cfg, const void* q, const void* k, const void* v,
                  void* pyr_q, void* pyr_k, void* pyr_v, double* sq, uint32_t* scale, void* stream);

/* (ii) Score, top-K descent, ordering. [LH] §3.1 stage (ii), Fig. 2 step 3,
 * Fig. 1 (topological sort into one causal sequence).
 * score(l,i) = max(sq[0], sq[1]). The coarsest level's entries are all
 * candidates; at each level l = L-1..1 the first k_l candidates in the order
 * (score desc, index asc) are expanded (radix select, or a chunked bitonic
 * sort in shared memory) and their p children become the next level's
 * candidates. The sub-sequence holds every candidate (LH_INCL_NESTED) or
 * every candidate that was not expanded (LH_INCL_PARTITION), ordered by
 * (last covered token, level) ascending (LH_ORDER_POST).
 * Outputs: sel (ascending indices, unused tail = -1), map, slot table.
 * ws: device workspace of at least plan.ws_bytes (contents not kept).
 * When L = 1, map is the identity and sel/slot/ws are not touched (may be NULL). */
lh_status lh_score_topk(const lh_config* cfg, const double* sq, int32_t* sel, int32_t* map,
                        int32_t* slot, void* ws, size_t ws_bytes, void* stream);

/* Dense gather: sub-sequence row j of xs = entry map[j] of x (level 0: the
 * token row of q/k/v; level >= 1: the pyramid row), in the attention operand
 * type: an exact copy for fp32 I/O; for bf16 I/O x * 2^-e in fp16 (e from the
 * head's row of `scale`, written by lh_pool), exact for every bf16 value within
 * 2^19 of the head's largest (a non-finite value is reported by
 * lh_get_device_error: LH_ERR_DEVICE, detail 102). fp16 gives the attention's P
 * and dS operands 11 significant bits instead of bf16's 8. [LH] Fig. 1 (dense
 * gather); "Lighthouse Attention Technique" (sort, then gather). */
lh_status lh_gather(const lh_config* cfg, const void* q, const void* k, const void* v,
                    const void* pyr_q, const void* pyr_k, const void* pyr_v, const int32_t* map,
                    const uint32_t* scale, void* qs, void* ks, void* vs, void* stream);

/* (iii) Causal attention on the sub-sequence, [LH] Eq. (1), scale 1/sqrt(D):
 * os = softmax(qs ks^T / sqrt(D) + causal mask) vs, lse = natural log of each
 * row's softmax denominator. bf16 I/O: tcgen05 tensor cores on the fp16
 * sub-sequence, P as fp16, fp32 accumulate; the operands' powers of two (from
 * `scale`) are taken out of the softmax scale and of os. fp32 I/O: fp32 SIMT
 * (`scale` unused). */
lh_status lh_attn_fwd(const lh_config* cfg, const void* qs, const void* ks, const void* vs,
                      const uint32_t* scale, float* os, float* lse, void* stream);

/* (iv) Scatter back, [LH] §3.1 stage (iv): token t of o receives, for every
 * sub-sequence entry covering t, that entry's row of os (weight 1), summed
 * coarse level first under cfg->accum, rounded to dtype. */
lh_status lh_scatter(const lh_config* cfg, const float* os, const int32_t* slot, void* o,
                     void* stream);

/* Backward of the scatter (adjoint, [LH] Fig. 1 gradient path): dos row j =
 * sum of dout over the tokens entry j covers (fp32, level by level), stored
 * as the backward operand type (fp16 for bf16 I/O: the block sums of pooled
 * entries need more significand than bf16 has; fp32 for fp32 I/O);
 * delta[j] = sum_d (stored block sum)[d] * os[j][d]. For bf16 I/O the stored
 * sums are sum * 2^-e with the head's exponent from its largest block sum,
 * recorded in row 3 of `scale` (a first pass records it; a second redoes the
 * heads that need e != 0). A non-finite block sum is reported by
 * lh_get_device_error (LH_ERR_DEVICE, detail 100). */
lh_status lh_scatter_bwd(const lh_config* cfg, const void* dout, const float* os,
                         const int32_t* slot, void* dos, float* delta, uint32_t* scale, void* stream);

/* Backward of (iii): gradients of Eq. (1) with P recomputed from lse:
 * dvs = P^T dos, dP = dos vs^T, dS = P o (dP - delta), dqs = dS ks / sqrt(D),
 * dks = dS^T qs / sqrt(D). Deterministic (no atomics). bf16 I/O: tcgen05
 * kernels on the fp16 sub-sequence and fp16 dos, fp32 accumulate (dS feeding
 * dqs is split into an fp16 head and remainder), the operands' powers of two
 * (from `scale`) taken out of P, delta and the three results; fp32 I/O: SIMT
 * kernels. A non-finite dQ or dK (a dS beyond the fp16 range, or non-finite
 * data) is reported by lh_get_device_error (LH_ERR_DEVICE, detail 101). */
lh_status lh_attn_bwd(const lh_config* cfg, const void* qs, const void* ks, const void* vs,
                      const void* dos, const float* lse, const float* delta, const uint32_t* scale,
                      float* dqs, float* dks, float* dvs, void* stream);

/* Backward of gather + mean-pool ([LH] Fig. 1 gradient path): token t of dx
 * receives dxs[j] / p^l(j) for every entry j covering t, summed coarse first
 * under cfg->accum, rounded to dtype; for x in {q, k, v}. */
lh_status lh_spread(const lh_config* cfg, const float* dqs, const float* dks, const float* dvs,
                    const int32_t* slot, void* dq, void* dk, void* dv, void* stream);

/* Token-range forms of lh_pool and lh_scatter, for fusing the path with the
 * projections next to it ("Long Context Pre-Training with Lighthouse
 * Attention", Fig. 1: the Q/K/V projections feed the pyramid pool, the
 * scatter-back feeds the output projection). A caller that produces Q, K, V
 * chunk by chunk pools each chunk right after its projection wrote it, while
 * the chunk is still in L2, and scatters the output chunk by chunk just before
 * the output projection reads it. Only the tokens [t0, t0 + nt) of every
 * sequence are read (lh_pool_range) or written (lh_scatter_range), with the
 * pyramid entries, norms, slot table and sub-sequence rows at their places in
 * the whole problem's buffers; the results equal lh_pool / lh_scatter's for
 * those tokens bit for bit. t0 and nt: multiples of p^(L-1), t0 + nt <= N;
 * L >= 2. lh_pool_range accumulates the magnitude rows of `scale` over its
 * calls; the call with t0 == 0 resets them first, so cover a sequence in order
 * from its start. Errors as lh_pool / lh_scatter, LH_ERR_SHAPE for a bad range. */
lh_status lh_pool_range(const lh_config* cfg, int t0, int nt, const void* q, const void* k, const void* v,
                        void* pyr_q, void* pyr_k, void* pyr_v, double* sq, uint32_t* scale, void* stream);
lh_status lh_scatter_range(const lh_config* cfg, int t0, int nt, const float* os, const int32_t* slot, void* o,
                           void* stream);

/* Device buffers of one forward+backward, caller-owned (sizes from lh_plan). */
typedef struct {
  void *pyr_q, *pyr_k, *pyr_v;   /* [B][H][E][D] dtype */
  double* sq;                    /* [2][B][H][E] */
  int32_t *sel, *map, *slot;     /* [B][H][L-1][K], [B][H][S], [B][H][E] */
  void *qs, *ks, *vs;            /* [B][H][S][D] fp16 (bf16 I/O) or fp32 */
  float *os, *lse;               /* [B][H][S][D], [B][H][S] */
  void* ws; size_t ws_bytes;     /* plan.ws_bytes */
  void* dos; float* delta;       /* [B][H][S][D] fp16 (bf16 I/O) or fp32, [B][H][S] */
  float *dqs, *dks, *dvs;        /* [B][H][S][D] */
  uint32_t* scale;               /* [4][B][H] operand magnitudes (see the layouts above) */
} lh_buffers;

/* Whole forward: lh_pool, lh_score_topk, lh_gather, lh_attn_fwd, lh_scatter. */
lh_status lh_forward(const lh_config* cfg, const void* q, const void* k, const void* v, void* o,
                     const lh_buffers* bufs, void* stream);

/* Whole backward (after lh_forward with the same bufs): lh_scatter_bwd,
 * lh_attn_bwd, lh_spread. */
lh_status lh_backward(const lh_config* cfg, const void* dout, void* dq, void* dk, void* dv,
                      const lh_buffers* bufs, void* stream);

/* ---------------------------------------------------------------------------
 * Sequence-sharded (context-parallel) path. The pages train at 1M-token
 * context over 32 B200s with context parallelism ("Nous Research's
 * Lighthouse Attention Trains 1.69x Faster on Million-Token Contexts", key
 * points; "Lighthouse Attention Technique": past 100K context the model is
 * scaled with context parallelism). Here rank r of `world` holds tokens
 * [r n, (r+1) n) of every sequence, n = N / world a multiple of p^(L-1), so
 * each pyramid entry lies in one shard. `cfg` always describes the WHOLE
 * sequence (N = world * n); L >= 2. One step, with the collectives the caller
 * runs between the calls (NCCL over NVLink: the steps are stream-ordered and
 * never wait on another rank):
 *   lh_cp_pool                 shard's pyramid, squared norms sq_loc and magnitude
 *                              rows 0-2 of scale
 *   all-gather of sq_loc into sq_gathered [world][2][B][H][E_loc]; all-reduce
 *   (max) of rows 0-2 of scale (uint32: the bit patterns order like the values)
 *   lh_cp_assemble_sq          -> sq [2][B][H][E] of the whole sequence
 *   lh_score_topk              the whole selection, map and slot table (the same
 *                              on every rank: every rank runs the same descent)
 *   lh_cp_segment              -> slot_loc [B][H][E_loc] (this rank's entries;
 *                              values are slots of the whole sub-sequence) and
 *                              seg [B][H][2] int32 = (first slot, count) of this
 *                              rank's entries: one contiguous run, since the
 *                              sub-sequence is sorted by position (Fig. 1)
 *   lh_cp_gather               rows of qs, ks, vs [B][H][S][D] (S of the whole
 *                              sequence): this rank's segment, zero elsewhere
 *   all-reduce (sum) of ks and of vs: every rank then holds all key/value rows
 *   lh_cp_attn_fwd             the segment's rows of os, lse (queries of the
 *                              segment over all keys before them)
 *   lh_cp_scatter              the shard's output tokens
 * Backward:
 *   lh_cp_scatter_bwd          the segment's rows of dos, delta (other rows of
 *                              dos are set to zero) and row 3 of scale (this
 *                              rank's own: dO's exponent may differ per rank)
 *   lh_cp_attn_bwd             dqs for the segment's rows; dks, dvs for ALL rows:
 *                              the contribution of this rank's queries
 *   all-reduce (sum) of dks and of dvs
 *   lh_cp_spread               the shard's dq, dk, dv
 * Buffers named like the single-GPU ones have the same layouts, with the
 * shard's tokens ([B][n][H][D]) and entries (E_loc per (b, h)). The attention
 * steps need bf16 I/O (tensor-core kernels): LH_ERR_DTYPE otherwise. Errors:
 * LH_ERR_SHAPE also for world < 1, rank outside [0, world), L < 2, or shards
 * that are not whole coarsest blocks. */
typedef struct {
  int world, rank;
  int n_loc;                       /* tokens per rank */
  int E_loc;                       /* entries of levels >= 1 per rank and (b, h) */
  int lvl_off_loc[LH_MAX_LEVELS];  /* start of level l within E_loc (l >= 1) */
  lh_plan_t global;                /* plan of the whole sequence (S = rows of qs ... dvs) */
} lh_cp_plan_t;

lh_status lh_cp_plan(const lh_config* cfg, int world, int rank, lh_cp_plan_t* out);
lh_status lh_cp_pool(const lh_config* cfg, int world, int rank, const void* q, const void* k, const void* v,
                     void* pyr_q, void* pyr_k, void* pyr_v, double* sq_loc, uint32_t* scale, void* stream);
lh_status lh_cp_assemble_sq(const lh_config* cfg, int world, const double* sq_gathered, double* sq,
                            void* stream);
lh_status lh_cp_segment(const lh_config* cfg, int world, int rank, const int32_t* map, const int32_t* slot,
                        int32_t* slot_loc, int32_t* seg, void* stream);
lh_status lh_cp_gather(const lh_config* cfg, int world, int rank, const void* q, const void* k, const void* v,
                       const void* pyr_q, const void* pyr_k, const void* pyr_v, const int32_t* map,
                       const int32_t* seg, const uint32_t* scale, void* qs, void* ks, void* vs, void* stream);
lh_status lh_cp_attn_fwd(const lh_config* cfg, int world, int rank, const int32_t* seg, const void* qs,
                         const void* ks, const void* vs, const uint32_t* scale, float* os, float* lse,
                         void* stream);
lh_status lh_cp_scatter(const lh_config* cfg, int world, int rank, const float* os, const int32_t* slot_loc,
                        void* o, void* stream);
lh_status lh_cp_scatter_bwd(const lh_config* cfg, int world, int rank, const void* dout, const float* os,
                            const int32_t* slot_loc, const int32_t* seg, void* dos, float* delta, uint32_t* scale,
                            void* stream);
lh_status lh_cp_attn_bwd(const lh_config* cfg, int world, int rank, const int32_t* seg, const void* qs,
                         const void* ks, const void* vs, const void* dos, const float* lse, const float* delta,
                         const uint32_t* scale, float* dqs, float* dks, float* dvs, void* stream);
lh_status lh_cp_spread(const lh_config* cfg, int world, int rank, const float* dqs, const float* dks,
                       const float* dvs, const int32_t* slot_loc, void* dq, void* dk, void* dv, void* stream);

/* Reads and clears the device error word set by bounded waits and device
 * checks (LH_OK, LH_ERR_TIMEOUT or LH_ERR_DEVICE); *detail receives the
 * kernel-specific code (0 if none). Synchronises `stream`. */
lh_status lh_get_device_error(void* stream, int* detail);

/* Number of liblh kernels launched by this process so far. */
unsigned long long lh_launch_count(void);

/* Diagnostics (the pages have no counterpart: this checks the failure path).
 * Launches one warp that waits on an mbarrier nothing ever arrives on, through
 * the same bounded wait every kernel uses, with a bound of `limit_cycles` SM
 * clock cycles (1 .. 2e9). The wait gives up, the device error word records
 * LH_ERR_TIMEOUT with detail 900 (lh_get_device_error returns it), the kernel
 * ends normally and the context stays usable. `gave_up`: device int, set to 1
 * when the wait gave up. LH_ERR_NULL / LH_ERR_SHAPE for bad arguments, checked
 * before the launch. */
lh_status lh_selftest_timeout(long long limit_cycles, int* gave_up, void* stream);

/* Diagnostics (the pages have no counterpart: this checks an arithmetic
 * building block). The attention kernels compute part of each softmax tile's
 * exponentials 2^x with a polynomial on the FMA pipe instead of the
 * special-function unit's ex2.approx (range reduction to [-1/2, 1/2], degree-5
 * minimax polynomial, exponent added in the bit pattern; inputs below -125 give
 * 2^-125). This evaluates both on n device floats x: y_fma[i] from the
 * polynomial, y_sfu[i] from ex2.approx.ftz.f32. Device buffers of n floats.
 * LH_ERR_NULL / LH_ERR_SHAPE before any launch; LH_ERR_CUDA if the launch fails. */
lh_status lh_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int n, void* stream);

/* lh_score_topk without a caller workspace (the paper has no counterpart: this
 * is for callers, not the method). Some callers cannot provide or allocate a
 * device workspace: a fixed arena that owns all device memory and may not
 * grow, or a hot path that may not call cudaMalloc because it can synchronise
 * the device. This variant keeps the descent's scratch in a fixed 8 MiB device
 * array inside liblh, which every GPU that loads the library holds until the
 * process exits; nothing is allocated per call.
 * Same inputs, outputs, results and errors as lh_score_topk, plus
 * LH_ERR_WORKSPACE when the problem needs more scratch than the array holds
 * (plan.ws_bytes > 8 MiB, i.e. 5*B*H*(sum of m_l) > 2,097,152; checked before any launch).
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress), so make that first call before any stream capture;
 * the address is kept for the life of the process (see the note on
 * cudaDeviceReset at the top of this file).
 * All calls share the one array, and it keeps the previous call's contents
 * (every scratch word is written before it is read, so nothing needs
 * clearing). Calls that overlap on the GPU, from different streams or host
 * threads, race on it: serialise them. */
lh_status lh_score_topk_noalloc(const lh_config* cfg, const double* sq, int32_t* sel, int32_t* map,
                                int32_t* slot, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LH_H */
