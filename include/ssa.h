/*
 * ssa.h -- C ABI of libssa.so: content-routed block-sparse exact attention
 * on NVIDIA B200 (sm_100a).
 *
 * The operation (jonsmirl/ssa README, introduction and "Algorithm and
 * complexity"; SingleZombie/LLSA README, "Minimum Usage" for the non-causal
 * variant): keys are mean-pooled into blocks of Bk rows; every query block of
 * Bq rows scores the summaries of its admissible key blocks, keeps the top-k
 * (ties go to the lower block index), adds the local causal window of W
 * tokens, and runs ordinary exact softmax attention over that union only.
 * The dense N x N score matrix is never formed.
 *
 * Conventions for every entry point
 *   Layout     Q: bf16 [B, Hq, N, D]; K, V: bf16 [B, Hkv, N, D]; O like Q.
 *              Contiguous, row-major, D innermost.  Query head h reads KV
 *              head h / (Hq / Hkv).
 *   Pointers   Device pointers unless stated otherwise.  Q, K, V, O must be
 *              16-byte aligned (the kernels move them with TMA / 16-byte
 *              vectors); float and int32 buffers 16-byte aligned.
 *   Ownership  The caller owns every buffer.  The library allocates no device
 *              memory: its device state is a file-scope error word per device
 *              that ssa_check_error reads and clears, and the fixed scratch
 *              of ssa_forward_static.
 *   Streams    Every call is asynchronous on the caller's stream (a
 *              cudaStream_t passed as ssa_stream_t; NULL = legacy default
 *              stream).  Calls on one stream run in order.
 *   Errors     Argument errors are returned synchronously before any launch,
 *              with a message in ssa_last_error_message().  Launch failures
 *              return SSA_ERR_CUDA.  Device-side failures (a bounded wait
 *              that ran out, a failed bounds check) set the device error
 *              word; ssa_check_error() reports them.  Kernels never trap.
 *   Threading  Thread-safe; the last-error message is per host thread.
 */
#ifndef SSA_H_
#define SSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* ssa_stream_t; /* a cudaStream_t */

typedef enum {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = 1,  /* a size, pointer or alignment is invalid       */
  SSA_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement  */
  SSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required    */
  SSA_ERR_CUDA = 4,         /* a CUDA runtime call or a launch failed        */
  SSA_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out            */
  SSA_ERR_DEVICE_CHECK = 6  /* a device-side bounds/consistency check failed */
} ssa_status;

/* Method parameters.  Names follow the pages' notation. */
typedef struct {
  int32_t B;               /* batch                                            */
  int32_t Hq;              /* query heads                                      */
  int32_t Hkv;             /* key/value heads; Hq % Hkv == 0                   */
  int32_t N;               /* tokens; multiple of block_k and of block_q       */
  int32_t D;               /* head dim: 64 or 128                              */
  int32_t block_k;         /* Bk: key block, power of two in [16, 128]         */
  int32_t block_q;         /* Bq: query block, power of two in [16, 128]       */
  int32_t top_k;           /* k: routed blocks per query block, 0..64          */
  int32_t window;          /* W: local causal window in tokens (i-W < j <= i)  */
  int32_t causal;          /* 1 causal (requires W >= 1); 0 non-causal (W = 0, k >= 1) */
  float scale;             /* softmax scale; 0 -> 1/sqrt(D)                    */
  int32_t wait_timeout_us; /* bound on every device-side wait; 0 -> 2 s        */
  int32_t consensus;       /* 0: each query head attends over its own routed
                              blocks; 1: the query heads of a KV group share
                              one consensus list (ssa_route_consensus);
                              requires (Hq / Hkv) * top_k <= 512            */
  float beta;              /* weight of the second-cumulant routing term:
                              0 ranks by <qbar, mu_c> (ssa_route); otherwise
                              by <qbar, mu_c> + (beta/2) tr(Sigma_c Q2)
                              (ssa_route_features + ssa_route_cumulant)     */
  int32_t tree_fanout;     /* 0: flat routing (every admissible block scored).
                              F > 0: two-level routing (ssa_route_tree) with
                              F key blocks per super-block; a power of two in
                              [1, 256], at most N/Bk; requires beta == 0    */
  int32_t tree_beam;       /* two-level routing: super-blocks kept per query
                              block, 1..64 (0 when tree_fanout == 0)        */
} ssa_params;

/* Bytes of device workspace ssa_forward needs for these parameters:
 * K summaries, Q summaries, the routed index list and counts (plus the
 * consensus lists, the second-cumulant features and scores, or the
 * super-block summaries and kept super-blocks, when those options are on),
 * each 256-byte aligned.  Returns 0 if the parameters are invalid. */
size_t ssa_workspace_size(const ssa_params* p);

/* Block summary (step 1 of the path; jonsmirl/ssa README, "Algorithm and
 * complexity": mu_c, block c's mean key).
 *   x    bf16 [B, H, N, D] (device)
 *   out  fp32 [B, H, N / block, D] (device): out[..., c, :] = mean of rows
 *        c*block .. c*block + block - 1, summed in fp32 then scaled by
 *        1/block (exact: block is a power of two).
 * H is the head count of x (Hq for queries, Hkv for keys); block is Bk or Bq.
 * B, N and D are taken from p.  One kernel launch.
 * Non-finite inputs are outside the method's domain.  A summary with a NaN or
 * infinite entry is still written and is reported through ssa_check_error
 * (SSA_ERR_DEVICE_CHECK); ssa_forward reports it the same way.  Routing never
 * selects a block whose score is NaN (so a count may fall below
 * min(top_k, admissible blocks)), and the outputs of rows that read a
 * non-finite key or value are unspecified; no kernel waits on data, so
 * nothing hangs. */
ssa_status ssa_block_summary(const ssa_params* p, const void* x, int32_t H,
                             int32_t block, float* out, ssa_stream_t stream);

/* Routing (steps 2-3; jonsmirl/ssa README, "Algorithm and complexity": the
 * block score <q, mu_c>, here with the second-cumulant weight beta = 0).
 *   qsum fp32 [B, Hq, N/Bq, D], ksum fp32 [B, Hkv, N/Bk, D] (device)
 *   idx  int32 [B, Hq, N/Bq, top_k] (device, out): for each query block the
 *        selected key blocks in ascending order, padded with -1
 *   cnt  int32 [B, Hq, N/Bq] (device, out): number of selected blocks,
 *        min(top_k, |admissible|)
 * Admissible blocks: causal -- completed blocks ending at or before the
 * query block's first token, (c+1)*Bk <= qb*Bq; non-causal -- all blocks.
 * Scores are fp32 dot products of the summaries; the top_k largest win, ties
 * to the lower block index.  top_k == 0 writes cnt = 0 only.  One launch.
 * Requires p->beta == 0 (SSA_ERR_INVALID_ARG otherwise). */
ssa_status ssa_route(const ssa_params* p, const float* qsum, const float* ksum,
                     int32_t* idx, int32_t* cnt, ssa_stream_t stream);

/* ssa_route with caller scratch, the same result bit for bit.  Problems the
 * tensor-core form routes (at least 2^25 admissible (query block, key block)
 * pairs over all heads, or SSA_ROUTER=tc) split the key summaries once into
 * the scratch -- tiles of 128 blocks as bf16 hi / lo parts in the MMA layout,
 * and their norms -- instead of once per CTA and tile, and the route then
 * copies each tile in with one bulk copy (two launches).  Elsewhere the
 * scratch is unused and may be NULL.
 *   workspace  device, 256-byte aligned, >= ssa_route_workspace_size(p)
 *              bytes (SSA_ERR_WORKSPACE otherwise); contents undefined
 *              before and after.  ssa_forward keeps the same image in its
 *              own workspace.
 * ssa_route_workspace_size returns 0 for invalid params, beta != 0, or when
 * the fp32 form routes the problem. */
size_t ssa_route_workspace_size(const ssa_params* p);
ssa_status ssa_route_with_workspace(const ssa_params* p, const float* qsum, const float* ksum,
                                    int32_t* idx, int32_t* cnt, void* workspace,
                                    size_t workspace_bytes, ssa_stream_t stream);

/* Second-cumulant routing features (jonsmirl/ssa README, "Algorithm and
 * complexity": r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q with Sigma_c block
 * c's second cumulant).  A query block scores by the mean of its queries'
 * scores, <qbar, mu_c> + (beta/2) tr(Sigma_c Q2), Q2 = mean of q_i q_i^T over
 * the block, which is one dot product of the feature vectors written here:
 *   queries == 0 (keys, block = Bk):    [mu_c | vech(Sigma_c)]
 *   queries == 1 (queries, block = Bq): [qbar | (beta/2) w . vech(Q2)]
 * vech = the upper triangle d <= e, row by row; w = 1 on the diagonal, 2 off
 * it; Sigma_c = (1/block) sum (x - mu)(x - mu)^T.
 *   x    bf16 [B, H, N, D] (device)
 *   out  fp32 [B, H, N/block, F] (device), F = D + D(D+1)/2 (2144 for D = 64)
 * block is a power of two <= 128 dividing N.  One launch. */
ssa_status ssa_route_features(const ssa_params* p, const void* x, int32_t H, int32_t block,
                              int32_t queries, float* out, ssa_stream_t stream);

/* Routing on the second-cumulant score: s = qfeat . kfeat over the admissible
 * blocks (fp32), then the top_k of every query block (ties to the lower block
 * index), listed ascending, padded with -1, with their count -- the same
 * output as ssa_route.
 *   qfeat   fp32 [B, Hq, N/Bq, F], kfeat fp32 [B, Hkv, N/Bk, F] from
 *           ssa_route_features (device)
 *   scores  fp32 [B, Hq, N/Bq, N/Bk] (device scratch: the score matrix)
 *   idx/cnt as for ssa_route (device, out)
 * Two launches. */
ssa_status ssa_route_cumulant(const ssa_params* p, const float* qfeat, const float* kfeat,
                              float* scores, int32_t* idx, int32_t* cnt, ssa_stream_t stream);

/* Super-block summaries for two-level routing (jonsmirl/ssa README,
 * "Algorithm and complexity": a hierarchical router in place of the flat
 * block scan; the measured tree has fanout 16).  Super-block S covers key
 * blocks S*F .. S*F+F-1, F = p->tree_fanout, and is summarised by the mean of
 * its F*Bk keys, computed as the fp32 mean of its children's means (exact in
 * real arithmetic: every block has Bk keys).
 *   ksum   fp32 [B, Hkv, N/Bk, D] block means (device), from ssa_block_summary
 *   ksum2  fp32 [B, Hkv, NS, D] (device, out), NS = (N/Bk) / F complete
 *          super-blocks (a trailing partial super-block has no summary)
 * Requires p->tree_fanout >= 1.  One launch. */
ssa_status ssa_tree_summary(const ssa_params* p, const float* ksum, float* ksum2,
                            ssa_stream_t stream);

/* Two-level (fixed-beam tree) routing (jonsmirl/ssa README, "Algorithm and
 * complexity"; "Mathematical status": fixed-beam routing is not an exact
 * selector -- a block whose super-block is not kept is never scored).  For
 * query block qb with admissible blocks 0 .. A-1 (the rule of ssa_route):
 *   1. the complete admissible super-blocks 0 .. A/F - 1 are scored by
 *      <qbar, super-block mean> (fp32) and the best tree_beam are kept,
 *      ties to the lower index -- the flat router on ksum2 with block F*Bk;
 *   2. the candidates are the F children of every kept super-block and the
 *      frontier blocks (A/F)*F .. A-1; the top_k of them by <qbar, mu_c>
 *      (fp32), ties to the lower index, are selected.
 * With tree_beam >= A/F every block is a candidate and the result is
 * ssa_route's.
 *   qsum, ksum      as for ssa_route (device)
 *   ksum2           from ssa_tree_summary (device)
 *   sup_idx/sup_cnt int32 [B, Hq, N/Bq, tree_beam] and [B, Hq, N/Bq]
 *                   (device, out): the kept super-blocks ascending, padded
 *                   with -1, and their count min(tree_beam, A/F)
 *   idx/cnt         as for ssa_route (device, out)
 * Requires p->tree_fanout >= 1 and p->beta == 0.  The lower level checks
 * the upper level's lists as it reads them (count within min(tree_beam, A/F),
 * super-blocks ascending and complete); a failed check is reported through
 * ssa_check_error (SSA_ERR_DEVICE_CHECK) and the bad entry contributes no
 * candidates.  Two launches. */
ssa_status ssa_route_tree(const ssa_params* p, const float* qsum, const float* ksum,
                          const float* ksum2, int32_t* sup_idx, int32_t* sup_cnt, int32_t* idx,
                          int32_t* cnt, ssa_stream_t stream);

/* GQA-shared consensus route (jonsmirl/ssa README, "Complete 10M transformer
 * result": one route formed across heads by consensus, carrying the blocks
 * with the most votes; "Mathematical status": a highest-count reservoir keeps
 * the items the per-head selectors voted for most often).  Every query head
 * of a KV group votes once for each block of its own list; the group keeps
 * the first min(top_k, #voted blocks) blocks in the order (votes descending,
 * block index ascending) -- the method's lower-index tie rule.
 *   idx/cnt        per-head lists as written by ssa_route: int32
 *                  [B, Hq, N/Bq, top_k] and [B, Hq, N/Bq] (device)
 *   idx_kv/cnt_kv  int32 [B, Hkv, N/Bq, top_k] and [B, Hkv, N/Bq] (device,
 *                  out): the group's blocks ascending, padded with -1, and
 *                  their count.  KV head kv's group is query heads
 *                  kv*g .. kv*g + g - 1, g = Hq / Hkv.
 * Requires (Hq / Hkv) * top_k <= 512 (SSA_ERR_UNSUPPORTED otherwise).  Lists
 * with a count outside 0..top_k or a block outside 0..N/Bk-1 are reported
 * through ssa_check_error (SSA_ERR_DEVICE_CHECK) and the bad entries skipped.
 * One launch; p->consensus is not consulted. */
ssa_status ssa_route_consensus(const ssa_params* p, const int32_t* idx, const int32_t* cnt,
                               int32_t* idx_kv, int32_t* cnt_kv, ssa_stream_t stream);

/* Attend (step 4; jonsmirl/ssa README, introduction: ordinary softmax over
 * the selected keys; "Mathematical status": the routed set is cut at each
 * query's position).  For query i in query block qb the key set is
 *   causal:     {keys of idx[qb]} U {i-W < j <= i}, cut at j <= i
 *   non-causal: {keys of idx[qb]}
 * counted once each; o_i = softmax(scale * q_i . k_j) . v_j over the set.
 *   q, k, v  bf16 (device), layouts above
 *   idx/cnt  as written by ssa_route (any valid lists: ascending, distinct,
 *            admissible, cnt <= top_k); with p->consensus the per-group
 *            lists of ssa_route_consensus, [B, Hkv, N/Bq, top_k] and
 *            [B, Hkv, N/Bq], used by every query head of the group (the
 *            kernel then packs two heads of a group into one tile)
 *   o        bf16 [B, Hq, N, D] (device, out), round-to-nearest-even
 *   lse      fp32 [B, Hq, N] (device, out, may be NULL): natural-log
 *            log-sum-exp of the scaled logits over the key set
 * One launch of the fused TMA + tcgen05 kernel. */
ssa_status ssa_attend(const ssa_params* p, const void* q, const void* k, const void* v,
                      const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                      ssa_stream_t stream);

/* The whole path in one call: summaries of K and Q (one launch) and routing
 * -- or, with p->beta != 0, the second-cumulant features of K and Q and
 * ssa_route_cumulant --, or, with p->tree_fanout > 0, the super-block
 * summaries and ssa_route_tree --, (with p->consensus) the consensus route, attend.  workspace must hold
 * ssa_workspace_size(p) bytes (device, 256-byte aligned); when the flat route
 * takes the tensor-core form its last ssa_route_workspace_size(p) bytes hold
 * the router's pre-split key image (one more launch).  idx_out / cnt_out
 * (device, may be NULL) receive the lists attend used when given -- per head
 * [B, Hq, N/Bq, top_k], or per KV group [B, Hkv, N/Bq, top_k] with
 * p->consensus; otherwise they live in the workspace.  lse may be NULL. */
ssa_status ssa_forward(const ssa_params* p, const void* q, const void* k, const void* v,
                       void* o, float* lse, int32_t* idx_out, int32_t* cnt_out,
                       void* workspace, size_t workspace_bytes, ssa_stream_t stream);

/* ssa_forward without a workspace argument, for callers that cannot allocate
 * device memory at call time -- for example code running inside a host
 * framework's launch callback or plugin, where cudaMalloc is forbidden (it can
 * synchronise the device, is not allowed while a stream is being captured, and
 * bypasses the framework's own memory pool), or code with no allocator at all.
 * No counterpart on the pages: this is an interface convenience, not part of
 * the method.
 *
 * The scratch (K and Q summaries, routed lists, counts) is a fixed 32 MiB
 * array inside the library's device module; every device that loads the
 * library keeps it until the process exits.  Shapes whose ssa_workspace_size
 * exceeds 32 MiB (33554432 bytes) are rejected with SSA_ERR_WORKSPACE and
 * nothing is launched.  The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.  The first call on each device looks up the
 * scratch's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  The address is kept per
 * device and context: the first call after the device's context was made anew
 * (cudaDeviceReset, or the primary context released and retaken) looks it up
 * again, since the reloaded module may place the array elsewhere.  All calls
 * share the one
 * scratch, which keeps the previous call's contents (every byte the path reads
 * is rewritten first, so nothing needs clearing); calls that can overlap on the
 * GPU -- on different streams, or from different host threads -- race on it
 * and must be serialised by the caller.  Arguments and results are as for
 * ssa_forward. */
ssa_status ssa_forward_static(const ssa_params* p, const void* q, const void* k, const void* v,
                              void* o, float* lse, int32_t* idx_out, int32_t* cnt_out,
                              ssa_stream_t stream);

/* Bytes of device workspace ssa_attend_backward needs (0 if the parameters
 * are invalid): two fp32 per query row, the lists' transpose (one bit per
 * list head, 128-key tile and 64-query chunk: 235 MB for 14 heads at 1M
 * tokens, 0.23 MB at 32K) and, when Hq > Hkv, each query head's fp32 share
 * of dk and dv (2 * B * Hq * N * D * 4 bytes: 7.5 GB at 1M tokens). */
size_t ssa_backward_workspace_size(const ssa_params* p);

/* Backward of the read with the selection held fixed (jonsmirl/ssa README,
 * introduction: within a query's key set the read is ordinary softmax
 * attention; the routed lists are a discrete choice and pass no gradient).
 * For query i with key set S_i (the set ssa_attend reads), P_ij =
 * exp(scale q_i . k_j - lse_i) and upstream gradient g_i = dL/do_i:
 *   dv_j += P_ij g_i;  dS_ij = P_ij (g_i . v_j - delta_i), delta_i = g_i . o_i;
 *   dq_i = scale sum_j dS_ij k_j;  dk_j += scale dS_ij q_i.
 * A KV head's dk / dv sum over the query heads of its group.
 *   q, k, v, o  bf16 (device): the forward's inputs and output
 *   lse         fp32 [B, Hq, N] (device): the forward's log-sum-exp
 *   d_o         bf16 [B, Hq, N, D] (device): the upstream gradient
 *   idx/cnt     the lists the forward read (per head, or per KV group with
 *               p->consensus), as for ssa_attend
 *   dq          fp32 [B, Hq, N, D] (device, out)
 *   dk, dv      fp32 [B, Hkv, N, D] (device, out; every entry is written)
 *   workspace   ssa_backward_workspace_size(p) bytes (device, 256-byte aligned):
 *               delta and lse * log2(e) [B, Hq, N] fp32, the lists' transpose
 *               (one bit per list head, 128-key tile and 64-query chunk) and,
 *               when Hq > Hkv, every query head's share of dk and dv
 * The products run on the tensor cores (tcgen05, bf16 operands, fp32
 * accumulation in TMEM): a query-major kernel for dq over the forward's key
 * sets and a key-major kernel for dk / dv over the transposed lists.  P and
 * dS enter the MMAs as two bf16 parts each (hi + lo, about 16 significant
 * bits).  Every gradient is summed in a fixed order, so results are
 * reproducible bit for bit.  Launches: one memset (the transpose), delta,
 * the transpose (when top_k > 0), dq, dk / dv per (key tile, query head),
 * and (when Hq > Hkv) the sum of the heads' shares in head order.  The
 * environment variable SSA_BWD=simt selects the earlier CUDA-core form
 * instead (fp32 FMA, dk / dv cleared and accumulated with atomic adds, so
 * their last bits can vary).
 * List entries that are out of range, not ascending or not admissible are
 * reported through ssa_check_error (SSA_ERR_DEVICE_CHECK) and skipped. */
ssa_status ssa_attend_backward(const ssa_params* p, const void* q, const void* k, const void* v,
                               const void* o, const float* lse, const void* d_o,
                               const int32_t* idx, const int32_t* cnt, float* dq, float* dk,
                               float* dv, void* workspace, size_t workspace_bytes,
                               ssa_stream_t stream);

/* Bytes of device workspace ssa_decode needs for these parameters (0 if they
 * are invalid for decode). */
size_t ssa_decode_workspace_size(const ssa_params* p);

/* One decode step (jonsmirl/ssa README, introduction and "Algorithm and
 * complexity", for a single query): the query of every (b, query head) at
 * position i = n_ctx - 1 is its own query block.  It scores the completed
 * key blocks (c+1)*Bk <= i by <q, mu_c> (fp32), keeps the top_k (ties to the
 * lower block index), and reads exact softmax over the routed blocks' keys
 * united with the window i - W < j <= i (each key once).
 *   p          p->N is the cache capacity (a multiple of Bk); causal = 1,
 *              consensus = 0, beta = 0; block_q is not used
 *   q          bf16 [B, Hq, D] (device): the new queries
 *   k_cache,   bf16 [B, Hkv, N, D] (device): rows 0 .. n_ctx-1 valid, row
 *   v_cache    n_ctx - 1 holding the new token's key and value
 *   ksum_cache fp32 [B, Hkv, N/Bk, D] (device, in/out): block means.  Rows
 *              c < i/Bk - 1 must hold them on entry (ssa_block_summary over
 *              the prefilled cache, then earlier decode steps); the call
 *              writes row i/Bk - 1, the block that becomes admissible at i.
 *   o          bf16 [B, Hq, D] (device, out); lse fp32 [B, Hq] (nullable)
 *   idx_out    int32 [B, Hq, top_k] (nullable): the selection, ascending,
 *              -1 padded; cnt_out int32 [B, Hq] (nullable)
 *   workspace  ssa_decode_workspace_size(p) bytes (device, 256-byte aligned):
 *              the splits' partial lists and reads and one counter per
 *              (b, query head); nothing needs clearing between calls
 * Two launches: the routing splits, then the attend splits, of which the
 * last to finish for a head merges the splits' reads and writes o and lse. */
ssa_status ssa_decode(const ssa_params* p, const void* q, const void* k_cache, const void* v_cache,
                      int32_t n_ctx, float* ksum_cache, void* o, float* lse, int32_t* idx_out,
                      int32_t* cnt_out, void* workspace, size_t workspace_bytes,
                      ssa_stream_t stream);

/* Synchronise the stream, then read and clear this device's error word.
 * Returns SSA_OK, SSA_ERR_TIMEOUT, SSA_ERR_DEVICE_CHECK or SSA_ERR_CUDA. */
ssa_status ssa_check_error(ssa_stream_t stream);

/* Diagnostic: launch one block that waits, with the same bounded wait the
 * kernels use, on a barrier nothing ever arrives on; the wait gives up after
 * timeout_us microseconds and records SSA_ERR_TIMEOUT in the error word.
 * Lets a caller check the timeout path without a hang. */
ssa_status ssa_probe_wait_timeout(int32_t timeout_us, ssa_stream_t stream);

/* Measurement: one launch of n_ctas blocks of 256 threads, each thread
 * evaluating iters x 8 exponentials with the instruction the attend kernel's
 * softmax uses (ex2.approx.ftz.f32, in 8 independent chains y <- 2^-y).
 * Timing the launch gives the device's exponential rate, a ceiling of the
 * softmax: n_ctas * 256 * iters * 8 / seconds.  sink is a device float that
 * is never written in practice (the results only feed a branch that cannot
 * be taken); it must still be valid device memory. */
ssa_status ssa_probe_ex2_rate(int32_t n_ctas, int32_t iters, float* sink, ssa_stream_t stream);

const char* ssa_status_string(ssa_status s);
const char* ssa_last_error_message(void);
int32_t ssa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SSA_H_ */
