/*
 * cqsa.h -- C ABI of the CQS-decomposed exact attention library (libcqsa.so).
 *
 * The library computes exact softmax attention over one sequence by the CQS
 * Divide of Stream-CQSA: the N tokens are split into c = l(l-1)+1 chunks; the
 * c cyclic subsequences S_k = {(x + k) mod c : x in D} (D a perfect
 * difference set) each run masked attention so that every ordered chunk pair
 * is computed exactly once; each task emits local softmax statistics and a
 * log-sum-exp merge recomposes them into the full output.  Subsequences can
 * be divided again (recursion), and inputs held in pinned host memory are
 * streamed through a bounded device working set.
 *
 * Sources (page title, section):
 *   [A] "Stream-CQSA: Exact Out-of-Memory Recovery for Attention" (arXiv
 *       abstract page): recursive partition into independent subsequence
 *       tasks, recomposition of local statistics, exact output.
 *   [B] "Stream-CQSA: Breaking the Billion-Token Barrier on a Single GPU"
 *       (wispaper.ai blog): section "The CQS Divide" (c = l(l-1)+1, every
 *       chunk pair exactly once, Steiner system S(2,l,c)); section "The
 *       Recursive Benefit" (divide again until it fits); section
 *       "Implementation" (CQS mask, stream Q_i/K_i/V_i to the GPU, local
 *       numerators and denominators, aggregate); section "Performance"
 *       (host-device transfer overhead).
 *   [C] layerthelatestinalattice.com summary: subproblems sized to fit a
 *       stated memory budget; recomposition equals full attention.
 *
 * Conventions for every call:
 *   - Tensors q, k, v, out are [N, H, d] contiguous (one sequence, B = 1) in
 *     the plan's dtype; lse is fp32 [H, N], the natural log of the sum of
 *     exp(score) with score = <q_i, k_j> / sqrt(d).
 *   - The caller owns every tensor.  The plan owns its device arena, its
 *     streams and events; it never allocates device memory after the first
 *     forward call, and its arena never exceeds mem_budget_bytes when a
 *     budget is given.
 *   - No call aborts or exits.  Each returns a status; on failure
 *     cqsa_last_error() holds a message (thread-local).
 */
#ifndef CQSA_H
#define CQSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct cqsa_plan cqsa_plan_t; /* opaque; created by cqsa_plan*, freed by cqsa_plan_destroy */

typedef enum {
    CQSA_OK = 0,
    CQSA_ERR_INVALID_ARG = 1,       /* null pointer, bad size or option */
    CQSA_ERR_NO_DIFFERENCE_SET = 2, /* no perfect difference set of size l mod l(l-1)+1 (e.g. l = 7) */
    CQSA_ERR_BUDGET = 3,            /* no working set fits mem_budget_bytes */
    CQSA_ERR_NOT_PINNED = 4,        /* host mode given a pointer that is not page-locked host memory */
    CQSA_ERR_CUDA = 5,              /* a CUDA runtime call failed; message names it */
    CQSA_ERR_TIMEOUT = 6,           /* a bounded device-side wait ran out; the kernel stopped early */
    CQSA_ERR_UNSUPPORTED = 7,       /* valid request this build does not implement (e.g. d not 64/128) */
    CQSA_ERR_NO_DEVICE = 8,         /* no usable sm_100 device */
    CQSA_ERR_INTERNAL = 9           /* a consistency check failed (CQSA_DEBUG plan checks, injected faults) */
} cqsa_status_t;

typedef enum { CQSA_BF16 = 0, CQSA_FP32 = 1 } cqsa_dtype_t;

enum { CQSA_DEVICE = 0, CQSA_HOST = 1 };

/* How a device-mode forward recomposes the tasks' local statistics ([A]
 * recomposition; [B] "Implementation" step 4).
 *   CQSA_MERGE_SLOTS: every (task, query block) writes its partial O_j and
 *     lse_j to a slot; a merge kernel then takes the log-sum-exp over the
 *     slots.  The tasks' results are materialised as the pages describe.
 *     Up to 1024 partials per query block (levels 4, 3, 3 give 36; the
 *     merge stages a tile's lse values and weights in shared memory, with
 *     fewer rows per tile as the partials grow); beyond that cqsa_forward
 *     reports CQSA_ERR_UNSUPPORTED and the plan needs CQSA_MERGE_FUSED.
 *   CQSA_MERGE_FUSED: one CTA walks the allowed key blocks of all the tasks
 *     of its query rows; its online softmax is the merge, and it writes the
 *     output directly (no slots, no merge launch).
 * The streamed (host-mode) path always folds each task into a running
 * accumulator in the attention kernel's epilogue. */
typedef enum { CQSA_MERGE_SLOTS = 0, CQSA_MERGE_FUSED = 1 } cqsa_merge_t;

#define CQSA_MAX_LEVELS 4
#define CQSA_MAX_L 16

/* Full plan description.  levels >= 1 and l[0..levels-1] each >= 2; the
 * leaf block is ceil(N / prod_i (l_i (l_i - 1) + 1)) tokens (positions at or
 * past N belong to no pair, so N need not divide evenly).  1 <= N <=
 * 2^31 - 4096 (rows are 32-bit on the device).  mem_budget_bytes = 0 means
 * unlimited. */
typedef struct {
    int64_t N;
    int H;
    int d;
    int levels;
    int l[CQSA_MAX_LEVELS];
    int causal;
    int dtype; /* cqsa_dtype_t */
    size_t mem_budget_bytes;
    int merge; /* cqsa_merge_t; 0 (slots) when zero-initialised */
    int H_kv;  /* key/value heads (grouped-query attention): H must be a
                  multiple; query head h reads key/value head h / (H / H_kv).
                  0 = H.  k, v (and dk, dv) are then [N, H_kv, d]. */
    int B;     /* independent sequences per call (0 or 1: one): tensors are
                  [B, N, heads, d] and lse [B, H, N]; the sequences run one
                  after another through the plan on the call's stream. */
    int shard_rank;  /* task sharding over shard_count processes (0 or 1:
                        none): the plan's entries (leaf task, query block) go
                        to ranks by longest-first assignment of their allowed
                        pair counts, the same on every rank, and this plan
                        computes the entries of shard_rank with
                        cqsa_forward_partial (see there). */
    int shard_count;
    int host_tasks;  /* host mode: run the streamed forward task by task even
                        when every block of a head group fits the budget
                        (0: the resident schedule then, see
                        cqsa_plan_host_launch). */
} cqsa_plan_desc_t;

/* What a plan decided (for logging, tests and the benchmark). */
typedef struct {
    int64_t N;
    int H, d, levels, causal, dtype;
    int l[CQSA_MAX_LEVELS];
    int c[CQSA_MAX_LEVELS];
    int D[CQSA_MAX_LEVELS][CQSA_MAX_L]; /* difference set of each level */
    int64_t num_blocks;                 /* prod c_i */
    int64_t block_tokens;               /* N / num_blocks */
    int64_t num_tasks;                  /* leaf tasks = prod c_i */
    int64_t num_entries;                /* (leaf task, query block) pairs with >= 1 allowed key */
    int64_t max_slots;                  /* most partials any query block receives */
    int64_t max_task_rows;              /* tokens in the largest leaf task */
    int head_group;                     /* heads per streamed group in host mode */
    size_t device_arena_bytes;          /* arena of a device-mode forward */
    size_t host_arena_bytes;            /* arena of a host-mode forward (<= budget) */
    size_t h2d_bytes;                   /* planned host->device bytes of one host-mode forward */
    size_t d2h_bytes;                   /* planned device->host bytes of one host-mode forward */
    double useful_flops;                /* 4 N^2 H d, halved when causal */
    int merge;                          /* cqsa_merge_t of device-mode forwards */
    int H_kv;                           /* key/value heads */
    int B;                              /* sequences per call */
    int shard_rank, shard_count;        /* task sharding (count 1: none) */
    int64_t shard_entries;              /* entries this rank computes */
    int debug_checked;                  /* CQSA_DEBUG set: the plan passed the brute-force checks */
    double shard_pairs;                 /* allowed (query, key) pairs of those entries, per head */
    double total_pairs;                 /* allowed pairs of all entries, per head */
    int64_t cache_q_slots;              /* host mode: device block cache slots for query blocks */
    int64_t cache_kv_slots;             /* host mode: slots for key blocks (one in the K pool, one in the V pool) */
    int bwd_head_group;                 /* host-mode backward: heads per group (0: none fits the budget) */
    size_t bwd_host_arena_bytes;        /* arena of a host-mode backward (<= budget) */
    int64_t bwd_cache_slots;            /* host-mode backward: block slots of its device cache */
    size_t bwd_h2d_bytes;               /* planned host->device bytes of one host-mode backward */
    size_t bwd_d2h_bytes;               /* planned device->host bytes of one host-mode backward */
    size_t bwd_spill_host_bytes;        /* pinned host memory the host-mode backward takes for written-back sums */
    int64_t bwd_writebacks;             /* gradient-sum write-backs per head group (0: every block stays cached) */
    int host_resident;                  /* host-mode forward runs the resident schedule (1) or task by task (0) */
    int64_t host_launches;              /* launches of the resident schedule per head group (0: task by task) */
    int64_t arrival_blocks;             /* resident schedule: blocks per arrival group of the copy-in */
    int host_sets;                      /* resident schedule: head groups whose device buffers coexist
                                           (2: the next group's copies overlap this group's launches) */
} cqsa_plan_info_t;

/* One (leaf task, query block) entry of the work list, in global blocks. */
typedef struct {
    int64_t task;       /* leaf task index, planner order */
    int64_t q_block;    /* global query block */
    int64_t slot;       /* partial index of this entry among the query block's entries */
    int64_t num_runs;   /* runs of consecutive allowed key blocks */
    int64_t shard;      /* rank that computes this entry in a sharded plan (0 otherwise) */
} cqsa_entry_t;

/*
 * cqsa_plan -- plan attention over N tokens, H heads, head dim d, bf16.
 * Level 0 uses l; each further level uses max(3, l_prev - 1) ([B] "The
 * Recursive Benefit").  levels = 0 picks the fewest levels (<= 4) whose
 * host-mode working set fits mem_budget_bytes.  causal != 0 keeps keys at
 * or before the query position.  On success *out owns a new plan.
 * Host-only: touches no GPU.  Errors: INVALID_ARG, NO_DIFFERENCE_SET,
 * BUDGET, UNSUPPORTED.
 */
cqsa_status_t cqsa_plan(int64_t N, int H, int d, int l, int levels, int causal,
                        size_t mem_budget_bytes, cqsa_plan_t **out);

/* cqsa_plan_ex -- as cqsa_plan with per-level l and a dtype (bf16 or fp32). */
cqsa_status_t cqsa_plan_ex(const cqsa_plan_desc_t *desc, cqsa_plan_t **out);

/*
 * cqsa_forward -- run the planned attention ([A]; [B] "Implementation").
 *   host_or_device = CQSA_DEVICE: q, k, v, out, lse are device pointers on the
 *     current device.  Every task runs from HBM.  CQSA_MERGE_SLOTS plans write
 *     the tasks' partials to the plan's arena and one merge writes out and
 *     lse; CQSA_MERGE_FUSED plans write out and lse from the tile kernel.
 *   host_or_device = CQSA_HOST: all five are page-locked host pointers
 *     (cudaHostAlloc / pinned torch tensors).  Tasks are streamed: each
 *     task's missing Q/K/V blocks are copied into a device block cache on a
 *     copy stream, computed, folded into device-resident accumulators of the
 *     current head group in the kernel's epilogue, and finished blocks are
 *     copied back.  When every block of a head group fits the budget
 *     (info.host_resident), the resident schedule runs instead: each block
 *     is copied once per head group and each pair of blocks computed as soon
 *     as both have arrived (cqsa_plan_host_launch).
 *   stream: a cudaStream_t (0 = legacy default stream) the call is ordered
 *     after and that is ordered after all of its work.
 * Asynchronous: returns once all work is enqueued.  The first call on a plan
 * allocates its arena (one cudaMalloc, sized by the plan).  One forward at a
 * time per plan.  After that first call a device-mode forward (and likewise
 * cqsa_backward) enqueues only kernel launches on `stream`, so it may be
 * captured in a CUDA graph and replayed with new contents in the same
 * buffers; the streamed mode's internal streams and events are not for
 * capture.  Errors: INVALID_ARG, NOT_PINNED, CUDA, NO_DEVICE, BUDGET.
 * Device-side timeouts are reported by cqsa_plan_sync.
 */
cqsa_status_t cqsa_forward(cqsa_plan_t *plan, const void *q, const void *k,
                           const void *v, void *out, float *lse,
                           int host_or_device, void *stream);

/*
 * cqsa_backward -- gradients of the planned attention with respect to q, k,
 * v, given the forward's out and lse and the gradient dout of the loss with
 * respect to out.  The pages report the method's backward-gradient error and
 * forward-backward runtime ([A]) and backward memory ([B] "Precise
 * Scaling"); they do not spell the backward out.  Reading used here: with
 * the merged row statistics lse_i and D_i = <dout_i, out_i>, every allowed
 * (query, key) pair lies in exactly one task and contributes
 *     P = exp(s - lse_i),  dS = P (<dout_i, v_j> - D_i),
 *     dq_i += dS k_j / sqrt(d),  dk_j += dS q_i / sqrt(d),  dv_j += P dout_i
 * independently of the other pairs, so the tasks' partial gradients sum to
 * the exact gradients.
 *   Layouts: q, k, v, out, dout, dq, dk, dv [N, H, d] contiguous in the plan
 *     dtype; lse fp32 [H, N] as cqsa_forward wrote it.  The caller owns all.
 *   host_or_device = CQSA_DEVICE: all ten pointers on the current device.
 *   host_or_device = CQSA_HOST: all ten are page-locked host pointers, and
 *     the backward runs within the plan's mem_budget_bytes ([A]: forward and
 *     backward past the memory limit; [B] "Precise Scaling": the backward's
 *     peak memory).  Per group of cqsa_plan_info().bwd_head_group heads, the
 *     lse rows are copied up and D = rowsum(dout * out) is formed block by
 *     block; then the leaf tasks run in order, each bringing its missing
 *     blocks' Q, K, V, dout rows into a device block cache and adding its
 *     pairs' gradient terms into fp32 running sums kept beside them; a
 *     block's sums leave as the finished gradients after its last task.  When
 *     the cache holds fewer blocks than the sequence, an evicted block's sums
 *     are written back to pinned host memory the plan allocates
 *     (bwd_spill_host_bytes, not counted in the budget) and brought back for
 *     its next task (cqsa_plan_bwd_cache_task).  The first host-mode call
 *     allocates the backward's arena (bwd_host_arena_bytes); when the
 *     streamed forward's arena and this one would exceed the budget together,
 *     the other one is released first (and set up again by its next call).
 *     With grouped-query attention a head group holds whole key/value
 *     groups, and the key-stationary gradients run one launch per query
 *     head residue modulo the group size, so that the query heads of a
 *     group add into their key/value head's sums one launch at a time.
 *   CQSA_MERGE_SLOTS plans write each (task, query block) dq partial and
 *     each (task, key block) dk / dv partial to slots of a backward arena
 *     (allocated on the first call) and sum them; CQSA_MERGE_FUSED plans
 *     walk all the tasks of a block in one CTA and write dq, dk, dv directly.
 * Asynchronous on stream.  Errors: INVALID_ARG, NOT_PINNED, BUDGET,
 * UNSUPPORTED, CUDA, NO_DEVICE.
 */
cqsa_status_t cqsa_backward(cqsa_plan_t *plan, const void *q, const void *k, const void *v,
                            const void *out, const float *lse, const void *dout, void *dq, void *dk,
                            void *dv, int host_or_device, void *stream);

/*
 * Task sharding across processes (one GPU each).  The tasks of the CQS
 * Divide are independent ([A]; [B] "Implementation": each task's partial
 * result is aggregated afterwards), so a plan with shard_count = G splits
 * one problem's (task, query block) entries over G ranks and the ranks
 * exchange their log-sum-exp partials once:
 *   1. cqsa_forward_partial on every rank: o_r, lse_r of its entries.
 *   2. lse_max = max over ranks of lse_r          (all-reduce MAX, caller)
 *   3. cqsa_partial_rescale: w_r = exp(lse_r - lse_max), o_r *= w_r.
 *   4. o = sum over ranks of o_r, w = sum of w_r  (all-reduce SUM, caller)
 *   5. cqsa_partial_finish: out = o / w, lse = lse_max + ln w.
 * The collectives are the caller's (the Python binding uses NCCL through
 * torch.distributed); all arithmetic runs in this library's kernels.  Any
 * plan may run steps 1, 3 and 5 (with one rank they reproduce
 * cqsa_forward); cqsa_forward and cqsa_backward reject a plan with
 * shard_count > 1.  Device mode only; B sequences are handled as in
 * cqsa_forward (each buffer gains a leading B).
 */

/* cqsa_forward_partial -- this rank's part of the forward.  q, k, v as in
 * cqsa_forward (device pointers).  o_part fp32 [N, H, d] gets, for every row,
 * the attention over this rank's allowed keys normalised by its own
 * denominator (0 where it has none) and lse_part fp32 [H, N] the natural-log
 * denominator (-inf where it has none).  Caller-owned device buffers; the
 * first call allocates a small arena (work list, error word).  Asynchronous
 * on stream.  Errors: INVALID_ARG, CUDA, NO_DEVICE, UNSUPPORTED. */
cqsa_status_t cqsa_forward_partial(cqsa_plan_t *plan, const void *q, const void *k, const void *v,
                                   float *o_part, float *lse_part, void *stream);

/* cqsa_partial_rescale -- w[h][n] = exp(lse_part[h][n] - lse_max[h][n]) (0
 * when lse_part is -inf) and o_part[n][h][:] *= w[h][n], in place.  All fp32
 * device buffers laid out as in cqsa_forward_partial; w may not alias the
 * others.  Asynchronous on stream.  Errors: INVALID_ARG, CUDA. */
cqsa_status_t cqsa_partial_rescale(cqsa_plan_t *plan, float *o_part, const float *lse_part,
                                   const float *lse_max, float *w, void *stream);

/* cqsa_partial_finish -- out[n][h][:] = o_sum[n][h][:] / w_sum[h][n] in the
 * plan dtype and lse[h][n] = lse_max[h][n] + ln w_sum[h][n] (0 and -inf
 * where w_sum is 0).  Device buffers; out and lse as cqsa_forward writes
 * them.  Asynchronous on stream.  Errors: INVALID_ARG, CUDA. */
cqsa_status_t cqsa_partial_finish(cqsa_plan_t *plan, const float *o_sum, const float *w_sum,
                                  const float *lse_max, void *out, float *lse, void *stream);

/*
 * Owner exchange (the alternative to steps 2-5 above, and what the Python
 * binding uses by default).  Query block b belongs to rank
 * floor(b * G / num_blocks), so rank k owns the contiguous rows
 * [row_lo[k], row_lo[k + 1]).  Per sequence:
 *   2'. cqsa_shard_pack: for each rank k in order, for each block b that k
 *       owns and this rank has an entry for, in increasing b: o_part rows of
 *       b ([n_b][H][d] fp32) then lse_part of b ([H][n_b] fp32, padded to a
 *       multiple of four floats) into `send`.
 *   3'. all-to-all (caller): send_counts[k] floats to rank k; the received
 *       pieces concatenated in source-rank order (recv_counts[r] from r).
 *   4'. cqsa_shard_merge: for each row this rank owns, the log-sum-exp merge
 *       of its received partials ([A] recomposition) into `chunk`: out rows
 *       [rows_max][H][d] in the plan dtype, then lse [H][rows_max] fp32,
 *       each part padded to 16 bytes (chunk_bytes in all).
 *   5'. all-gather (caller): the G chunks in rank order.
 *   6'. cqsa_shard_unpack: out [N][H][d] and lse [H][N] from the chunks.
 * A block has entries on at most l ranks, so a rank sends about (l - 1) / G
 * of the partial rows rather than all of them twice; the all-gather moves the
 * output once, in the plan dtype.  All four calls take one sequence; device
 * pointers on the current device; asynchronous on stream.
 */

/* cqsa_shard_layout -- host only: send_counts[G], recv_counts[G] (fp32
 * values to and from each rank), row_lo[G + 1], *rows_max and *chunk_bytes
 * of this rank's plan.  Errors: INVALID_ARG. */
cqsa_status_t cqsa_shard_layout(cqsa_plan_t *plan, int64_t *send_counts, int64_t *recv_counts, int64_t *row_lo,
                                int64_t *rows_max, size_t *chunk_bytes);

/* cqsa_shard_pack -- step 2': o_part fp32 [N, H, d], lse_part fp32 [H, N]
 * (cqsa_forward_partial's outputs for one sequence) into send (fp32, the sum
 * of send_counts).  Errors: INVALID_ARG, CUDA. */
cqsa_status_t cqsa_shard_pack(cqsa_plan_t *plan, const float *o_part, const float *lse_part, float *send,
                              void *stream);

/* cqsa_shard_merge -- step 4': recv (fp32, the sum of recv_counts, as the
 * all-to-all left it) into chunk (chunk_bytes).  The first call allocates a
 * small table of the owned blocks' partial offsets.  Errors: INVALID_ARG,
 * UNSUPPORTED (a block with partials from more than 32 ranks), CUDA. */
cqsa_status_t cqsa_shard_merge(cqsa_plan_t *plan, const float *recv, void *chunk, void *stream);

/* cqsa_shard_unpack -- step 6': the G chunks (G * chunk_bytes, rank order)
 * into out [N, H, d] (plan dtype) and lse [H, N] fp32.  Errors:
 * INVALID_ARG, CUDA. */
cqsa_status_t cqsa_shard_unpack(cqsa_plan_t *plan, const void *chunks, void *out, float *lse, void *stream);

/* cqsa_backward_partial -- this rank's part of the backward of a sharded
 * plan (any plan: with one rank it is the whole backward).  Every allowed
 * pair's gradient terms depend only on the pair and the row statistics
 * (see cqsa_backward), so each rank sums the terms of its own entries and
 * one all-reduce SUM over ranks gives the gradients:
 *   q, k, v, out, lse, dout as for cqsa_backward (out and lse the full
 *   forward's, e.g. from the sharded exchange, on every rank);
 *   dq_part fp32 [N, H, d], dk_part, dv_part fp32 [N, H_kv, d]: this rank's
 *   sums (0 where it has no pair).  Device buffers owned by the caller.
 * The first call allocates the rank's backward arena.  Asynchronous on
 * stream.  Errors: INVALID_ARG, CUDA, NO_DEVICE. */
cqsa_status_t cqsa_backward_partial(cqsa_plan_t *plan, const void *q, const void *k, const void *v,
                                    const void *out, const float *lse, const void *dout, float *dq_part,
                                    float *dk_part, float *dv_part, void *stream);

/* cqsa_partial_cast -- count fp32 values (e.g. all-reduced gradient sums) to
 * the plan dtype, rounded to nearest even.  Device buffers; asynchronous on
 * stream.  Errors: INVALID_ARG, CUDA. */
cqsa_status_t cqsa_partial_cast(cqsa_plan_t *plan, const float *src, void *dst, int64_t count, void *stream);

/* cqsa_plan_sync -- wait for the plan's work on `stream` and report any
 * device-side error word (CQSA_ERR_TIMEOUT) raised since the last sync; the
 * message (cqsa_last_error) names the kernels whose wait ran out: device
 * forward, streamed forward, backward, partial forward or partial backward. */
cqsa_status_t cqsa_plan_sync(cqsa_plan_t *plan, void *stream);

/* cqsa_plan_info -- copy what the plan decided into *info. */
cqsa_status_t cqsa_plan_info(const cqsa_plan_t *plan, cqsa_plan_info_t *info);

/* cqsa_plan_task_blocks -- global blocks of leaf task t in increasing order
 * (its token sequence) and its subsequence index per level.  blocks must
 * hold max_blocks entries, path CQSA_MAX_LEVELS; *num_blocks gets the
 * count.  INVALID_ARG when t is out of range or max_blocks is too small. */
cqsa_status_t cqsa_plan_task_blocks(const cqsa_plan_t *plan, int64_t t, int64_t *blocks,
                                    int64_t max_blocks, int64_t *num_blocks, int *path);

/* cqsa_plan_cache_task -- the streamed path's device block cache as planned
 * for leaf task t (replayed for every head group; [B] "Implementation":
 * stream the blocks a subsequence needs).  Copies issued before the task's
 * kernel, in order: kinds[i] 0 for a query block (Q pool) or 1 for a key
 * block (K and V pools, same slot), blocks[i] the global block, slots[i] the
 * pool slot.  Slots the task's kernel reads, for each of its blocks in
 * cqsa_plan_task_blocks order: q_slot[m] and kv_slot[m] (-1: not read).
 * The plan never lets task t's copies evict a block task t - 1 reads (its
 * kernel may still run); the scheduler makes a copy wait for the kernel of
 * task t - 2 and, at a head-group boundary, for the previous kernel.
 * Arrays hold max_copies / max_blocks entries; *num_copies / *num_blocks
 * get the counts (arrays may be NULL to ask for the counts).  INVALID_ARG
 * when t is out of range or an array is too small; BUDGET when the plan has
 * no host-mode sizing.  A plan with info.host_resident set runs the resident
 * schedule instead (cqsa_plan_host_launch); this is then the cache the
 * task-by-task schedule would use with every block cached. */
cqsa_status_t cqsa_plan_cache_task(const cqsa_plan_t *plan, int64_t t, int32_t *kinds, int64_t *blocks,
                                   int32_t *slots, int64_t max_copies, int64_t *num_copies, int32_t *q_slot,
                                   int32_t *kv_slot, int64_t max_blocks, int64_t *num_blocks);

/* cqsa_plan_bwd_cache_task -- the host-mode backward's device block cache as
 * planned for leaf task t (replayed for every head group).  A slot holds one
 * block's Q, K, V and dO rows and its running dQ, dK, dV sums.  Copies issued
 * before the task's kernels, in order: block blocks[i] goes into slot
 * slots[i]; evicts[i] is the unfinished block whose sums are first written
 * back to host memory from that slot (-1: none); reloads[i] is 1 when the
 * block's sums come back from host memory, 0 when they start at zero.
 * member_slot[m]: the slot of the task's m-th block (cqsa_plan_task_blocks
 * order; -1 when the backward does not use it).  fin_blocks[j] /
 * fin_slots[j]: the blocks whose last task is t; after its kernels their
 * sums become the gradients (plan dtype) and go to the host.  The plan keeps
 * the blocks of task t - 1, and the slots of blocks it finished, out of task
 * t's copies.  Arrays may be NULL to ask for the counts.  INVALID_ARG when t
 * is out of range or an array is too small; BUDGET when no host-mode
 * backward fits the budget. */
cqsa_status_t cqsa_plan_bwd_cache_task(const cqsa_plan_t *plan, int64_t t, int64_t *blocks, int32_t *slots,
                                       int64_t *evicts, int32_t *reloads, int64_t max_copies, int64_t *num_copies,
                                       int32_t *member_slot, int64_t max_blocks, int64_t *num_blocks,
                                       int64_t *fin_blocks, int32_t *fin_slots, int64_t max_fin, int64_t *num_fin);

/* cqsa_plan_host_launch -- launch i (0 <= i < info.host_launches) of the
 * streamed forward's resident schedule, used when every block of a head
 * group fits the budget ([B] "Implementation": stream the blocks the tasks
 * need; here each block crosses the host link once per head group).  The
 * blocks are copied in increasing order; the copy stream marks every
 * info.arrival_blocks consecutive blocks.  With info.host_sets = 2 the
 * head groups alternate between two sets of device buffers, so one group's
 * copies run while the previous group's launches do; a group waits only for
 * the group before last (the same set).  Each set has its own two internal
 * compute streams, so the launches of consecutive groups also overlap.  The
 * launch waits for the mark of the group holding *need (the last block it
 * reads), runs on its set's compute stream *stream (0 or 1), and first
 * waits for launch *after of the other stream (-1: none).  It takes the plan's (query block, key block)
 * pairs pairs[2p], pairs[2p + 1], p < *num_pairs, in query-block order;
 * flags[p] is its entry's SEG flags for that query block (1: the block's
 * first launch, starts its accumulator; 2: its last, writes its finished
 * rows, which then go to the host).  Arrays may be NULL to ask for the
 * count.  INVALID_ARG when i is out of range or an array is too small. */
cqsa_status_t cqsa_plan_host_launch(const cqsa_plan_t *plan, int64_t i, int64_t *need, int32_t *stream,
                                    int32_t *after, int64_t *pairs, int32_t *flags, int64_t max_pairs,
                                    int64_t *num_pairs);

/* cqsa_plan_entry -- entry i (0 <= i < num_entries) of the work list and its
 * key runs: runs[2r], runs[2r+1] are the first and last global key block of
 * run r (inclusive).  runs must hold 2 * max_runs values. */
cqsa_status_t cqsa_plan_entry(const cqsa_plan_t *plan, int64_t i, cqsa_entry_t *entry,
                              int64_t *runs, int64_t max_runs);

/* cqsa_difference_set -- the lexicographically first perfect difference set
 * of size l modulo l(l-1)+1 that contains 0 and 1 ([B] "The CQS Divide";
 * [A] cyclic quorum sets).  D must hold l ints.  NO_DIFFERENCE_SET if none. */
cqsa_status_t cqsa_difference_set(int l, int *D);

/* cqsa_plan_debug -- failure-detection hooks for tests.  timeout_ns bounds
 * every device-side wait (0 restores the default of 4 s); stall_mma != 0
 * makes the bf16 kernel's MMA issuer issue nothing, so that the other
 * warps' bounded waits run out and the next cqsa_plan_sync reports
 * CQSA_ERR_TIMEOUT.  Never needed in normal use. */
cqsa_status_t cqsa_plan_debug(cqsa_plan_t *plan, uint64_t timeout_ns, int stall_mma);

/* cqsa_debug_inject -- host-side fault injection for tests.  kind =
 * CQSA_FAULT_ALLOC: the nth following device allocation of the library
 * (plan arenas) fails as if cudaMalloc had run out of memory; kind =
 * CQSA_FAULT_COPY: the nth following host<->device copy of a streamed
 * forward fails; kind = CQSA_FAULT_SETUP: the nth following upload of a
 * plan's tables (work lists, slot counts) into a freshly allocated arena
 * fails.  The failing call returns CQSA_ERR_CUDA without touching the GPU;
 * work already enqueued completes, and the plan stays usable (a setup that
 * failed part-way releases its arena, and the next call sets it up again).
 * nth = 0 clears; the setting is process-wide and fires once.  Errors:
 * INVALID_ARG. */
enum { CQSA_FAULT_ALLOC = 1, CQSA_FAULT_COPY = 2, CQSA_FAULT_SETUP = 3 };
cqsa_status_t cqsa_debug_inject(int kind, int64_t nth);

/* Per-kernel device time of a plan's launches, from CUDA events recorded
 * on the stream each kernel is launched on. */
typedef struct {
    int64_t attn_launches;  /* tile-attention kernel launches */
    int64_t merge_launches; /* log-sum-exp merge kernel launches */
    double attn_ms;         /* summed device time of those launches */
    double merge_ms;
    int64_t bwd_launches;   /* backward gradient kernel launches (dq and dk/dv) */
    double bwd_ms;
} cqsa_kernel_stats_t;

/* cqsa_plan_profile -- enable != 0: from the next forward on, record a CUDA
 * event pair around every kernel the plan launches (a few microseconds per
 * launch).  enable = 0 stops recording. */
cqsa_status_t cqsa_plan_profile(cqsa_plan_t *plan, int enable);

/* cqsa_plan_kernel_stats -- wait for the recorded events, add their times to
 * the plan's totals and copy the totals into *stats; reset != 0 then clears
 * the totals.  CUDA on an event failure. */
cqsa_status_t cqsa_plan_kernel_stats(cqsa_plan_t *plan, cqsa_kernel_stats_t *stats, int reset);

/* Size of the fixed device scratch array behind cqsa_forward_noalloc. */
#define CQSA_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * cqsa_forward_noalloc -- the device-resident forward without any device
 * allocation.  The pages have no counterpart: this is a convenience of this
 * library for callers that must not call cudaMalloc at call time (a
 * framework whose caching allocator already reserved the free device
 * memory, a process at its device-memory cap, or a loop that cannot afford
 * cudaMalloc's implicit device synchronisation).
 *   q, k, v, out: device pointers, [N, H, d] in the plan's dtype; lse: fp32
 *   [H, N] on the device; all five on the current device, which must be the
 *   plan's device if the plan was used before.  The caller owns them.  The
 *   task partials, work list and error word live in one file-scope device
 *   array of CQSA_NOALLOC_SCRATCH_BYTES (64 MiB) per device, held until the
 *   process exits.
 *   Set-up: the first call on a device looks up the array's address
 *   (cudaGetSymbolAddress), which loads the library's device code there and
 *   with it reserves the 64 MiB (under lazy module loading, the CUDA
 *   default, not earlier).  Make that first call early, while 64 MiB are
 *   still free (it fails with CQSA_ERR_CUDA otherwise), and before any stream
 *   capture.  Later calls on that device reserve and allocate nothing.
 *   Limits: the plan's partials (max_slots * N * H * d * 4 bytes, plus lse)
 *   and work list must fit the array; otherwise CQSA_ERR_BUDGET with the
 *   sizes in the message, and cqsa_forward is the way.  A CQSA_MERGE_FUSED
 *   plan runs as a slots plan here (partials in the array, then the merge),
 *   so plans with more than 1024 partials per query block are refused with
 *   CQSA_ERR_UNSUPPORTED, as are batched (B > 1), grouped-query and sharded
 *   plans.
 *   Calls share the array and keep the last call's contents; host callers
 *   are serialised, but work of two calls that overlaps on the GPU would
 *   race, so every call waits until its own work on `stream` has finished
 *   before returning, and then reports CQSA_ERR_TIMEOUT if a bounded device
 *   wait ran out.  Calls no cudaMalloc, cudaFree or other allocating
 *   routine.  Errors: INVALID_ARG, NO_DEVICE, BUDGET, UNSUPPORTED, CUDA,
 *   TIMEOUT.
 */
cqsa_status_t cqsa_forward_noalloc(cqsa_plan_t *plan, const void *q, const void *k,
                                   const void *v, void *out, float *lse, void *stream);

/* cqsa_plan_destroy -- free the plan, its arena, streams and events.  Waits
 * for the plan's outstanding work first.  Null is ignored. */
void cqsa_plan_destroy(cqsa_plan_t *plan);

/* cqsa_last_error -- message of the last failing call on this thread. */
const char *cqsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* CQSA_H */
