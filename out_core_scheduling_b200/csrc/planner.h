// planner.h -- host-side CQS planner: difference sets, subsequence tasks,
// CQS masks, recursion, work lists and memory sizing.  Pure C++ (no CUDA).
//
// Follows "Stream-CQSA: Breaking the Billion-Token Barrier on a Single GPU"
// (wispaper.ai blog): section "The CQS Divide" (c = l(l-1)+1 chunks, c
// subsequences of l chunks, every chunk pair exactly once), section "The
// Recursive Benefit" (divide a subsequence again), section "Implementation"
// (CQS mask against redundant work in overlapping chunks; stream each task's
// Q_i, K_i, V_i), and the layerthelatestinalattice.com summary (subproblems
// sized to a memory budget).
#pragma once
#include <stddef.h>
#include <stdint.h>

#include <algorithm>
#include <string>
#include <vector>

#include "worklist.h"

namespace cqsa {

constexpr int kMaxLevels = 4;
constexpr int64_t kMaxN = (1LL << 31) - 4096;  // 32-bit rows plus a unit or tile width

struct Level {
    int l = 0;            // chunks per subsequence
    int c = 0;            // chunks = l(l-1)+1
    std::vector<int> D;   // perfect difference set mod c
};

struct Leaf {
    std::vector<int> path;                  // subsequence index per level
    std::vector<int64_t> blocks;            // global blocks, increasing
};

struct KeyRun {
    int64_t b0, b1;                         // global key blocks, inclusive
    int32_t m0;                             // leaf member index of b0
};

struct Entry {
    int64_t task;                           // leaf index
    int64_t qb;                             // global query block
    int32_t mq;                             // leaf member index of qb
    int64_t slot;                           // partial index for qb
    std::vector<KeyRun> runs;
};

// Work list for one launch domain (device mode: the whole sequence; host
// mode: one leaf task in its local buffers).
struct WorkList {
    std::vector<WlEntry> entries;
    std::vector<WlRun> runs;
    std::vector<WlUnit> units;
};

struct PlanSpec {
    int64_t N = 0;
    int H = 0, d = 0;
    int levels = 0;
    int l[kMaxLevels] = {0, 0, 0, 0};
    int causal = 0;
    int elem_bytes = 2;                     // 2 = bf16, 4 = fp32
    size_t budget = 0;                      // 0 = unlimited
    int fused = 0;                          // device mode: merge in the kernel, no partial slots
    int Hkv = 0;                            // key/value heads (grouped-query attention); 0 = H
    int B = 1;                              // independent sequences of N tokens per call
    int shard_rank = 0, shard_count = 1;    // task sharding over processes
    int host_tasks = 0;                     // streamed forward: task by task even when every block fits
    int kv_group() const { return H / (Hkv > 0 ? Hkv : H); }
    // Key/value heads a streamed head group of g query heads reads.
    int kv_heads_of(int g) const { return g >= kv_group() ? g / kv_group() : 1; }
};

// Device block cache of the streamed path.  A Q slot holds one query block
// of the current head group ([block, g, d]); a KV slot holds its K and V
// blocks (same slot index in the K pool and the V pool, so one key
// coordinate addresses both).  The task order is fixed, so the cache is
// simulated at plan time with Belady's rule (evict the block whose next use
// is farthest away); blocks of the current and the previous task are never
// evicted, because the previous task's kernel may still be reading them.
struct PoolCopy {
    int32_t kind;     // 0: Q block, 1: K and V blocks
    int64_t block;    // global block
    int32_t slot;
};

struct PoolPlan {
    int64_t q_slots = 0, kv_slots = 0;
    std::vector<std::vector<PoolCopy>> copies;          // per leaf task, in copy order
    std::vector<std::vector<int32_t>> q_slot, kv_slot;  // per leaf task, per member; -1: unused
    int64_t q_copies = 0, kv_copies = 0;                // per head group
};

// Device block cache of the streamed backward.  A slot holds one block of
// the current head group: its Q, K, V and dO rows ([block, g, d] each, the
// plan dtype) and its running dQ, dK and dV sums ([block, g, d] fp32 each).
// A block's sums start at zero on its first task, collect the terms of every
// task that contains it, and leave as the finished gradients after its last
// task.  The task order is fixed, so the cache is simulated at plan time
// with Belady's rule; a block evicted between two of its tasks has its
// sums written back to host memory and brought back on its next task.
// Blocks of the current and the previous task stay (the previous task's
// kernels may still run), and so does the slot of a block finished by the
// previous task (its gradients may still be on their way to the host).
struct BwdCopy {
    int64_t block;    // global block brought into `slot`
    int32_t slot;
    int64_t evict;    // unfinished block written back from `slot` first (-1: none)
    int32_t reload;   // 1: the block's sums come back from host memory; 0: they start at zero
};

struct BwdCachePlan {
    int64_t slots = 0;
    std::vector<std::vector<BwdCopy>> copies;                      // per leaf task, in copy order
    std::vector<std::vector<int32_t>> member_slot;                 // per leaf task, per member
    std::vector<std::vector<std::pair<int64_t, int32_t>>> finals;  // per leaf task: (block, slot) finished by it
    int64_t loads = 0, writebacks = 0;                             // per head group
};

struct BwdSizing {
    int head_group = 0;     // 0: no streamed backward fits the budget
    size_t arena = 0;       // device bytes
    int64_t slots = 0;
    size_t h2d = 0, d2h = 0;
    size_t spill_host = 0;  // pinned host bytes for written-back sums (0: none needed)
};

// Exchange of a sharded forward to the query blocks' owners.  Query block b
// belongs to rank floor(b * G / num_blocks), so each rank owns a contiguous
// range of rows.  A rank sends, to each owner in rank order, the partials
// (o rows [n_b][H][d] fp32, then lse [H][n_b] fp32 padded to a multiple of
// four floats) of the owner's blocks it
// has an entry for, in increasing block order; the owner merges the
// partials it receives (sources in rank order) and the ranks all-gather the
// merged rows.
struct ShardPiece {
    int64_t block;
    int64_t offset;  // floats into the send (or receive) buffer
};

struct ShardLayout {
    int G = 1, me = 0;
    std::vector<int32_t> owner;                 // per block
    std::vector<int64_t> row_lo;                // G + 1: rows [row_lo[k], row_lo[k + 1]) belong to rank k
    int64_t rows_max = 0;                       // most rows a rank owns
    std::vector<int64_t> send_counts, recv_counts;  // floats to / from each rank
    std::vector<ShardPiece> send;               // this rank's pieces, in send order
    int64_t own_first = 0, own_count = 0;       // this rank's blocks [own_first, own_first + own_count)
    std::vector<std::vector<int64_t>> own_offsets;  // per owned block: its partials' receive offsets
    size_t out_bytes = 0, chunk_bytes = 0;      // gathered chunk: out rows, then lse [H][rows_max]
};

struct Sizing {
    int head_group = 0;
    size_t host_arena = 0;
    size_t device_arena = 0;
    size_t h2d = 0, d2h = 0;
    int64_t q_slots = 0, kv_slots = 0;
    bool resident = false;  // the streamed forward runs the resident schedule (HostLaunch)
    int sets = 1;           // resident schedule: head groups whose buffers coexist (copies of the next overlap this one)
};

// Streamed forward when the device holds every block of a head group at
// once (the resident schedule).  The blocks are copied in increasing order,
// block b to pool rows [b * block, ...), and the copy stream marks each
// arrival group of consecutive blocks.  A launch takes the plan's (query
// block, key block) pairs whose blocks have arrived: one entry per query
// block with the union of those pairs' key blocks as maximal runs, folded
// into the block's running accumulator by the epilogue merge; the launch
// that takes a query block's last pairs writes its finished rows.  Every
// pair of every entry of the plan is taken exactly once.  While blocks
// arrive, launch pairs come in two kinds per arrival group k: the new
// query blocks of group k against keys of groups <= k, and the query
// blocks of earlier groups against the keys of group k.  Pairs that need
// one of the last arrival groups are taken a few query groups at a time
// (enough for two launches in flight to cover the SMs; groups ready at the
// same arrival only, longest key chains first), so that finished rows go
// to the host while the rest still computes.
// Launches alternate between two compute streams; a launch waits for the
// latest launch on the other stream that touched one of its query blocks
// (launches on one stream run in order), so the merges of a query block
// happen in launch order and launches of disjoint query blocks overlap.
struct HostLaunch {
    WorkList wl;                  // global rows (slot b holds block b)
    int64_t need = 0;             // last block it reads
    int32_t stream = 0;           // compute stream 0 or 1
    int32_t after = -1;           // launch on the other stream it waits for (-1: none)
    std::vector<int64_t> finish;  // query blocks whose rows it finishes, increasing
};

class Planner {
public:
    // Returns "" on success, else an error message; *code gets a status.
    std::string build(const PlanSpec &spec, int *code);

    PlanSpec spec;
    std::vector<Level> levels;
    int64_t num_blocks = 0;     // prod c_i
    int64_t block = 0;          // tokens per block: ceil(N / num_blocks)
    // Token rows of block b: [b * block, block_end(b)); blocks at or past N
    // hold none (N need not be a multiple of num_blocks).
    int64_t block_end(int64_t b) const { return std::min<int64_t>((b + 1) * block, spec.N); }
    int64_t block_rows(int64_t b) const { return std::max<int64_t>(0, block_end(b) - b * block); }
    std::vector<Leaf> leaves;
    std::vector<Entry> entries; // ordered by (task, qb)
    std::vector<int32_t> slots_per_block;
    int64_t max_slots = 0;
    int64_t max_task_rows = 0;
    Sizing sizing;
    // Task sharding: the rank of each entry (longest-first assignment of
    // the entries' allowed pair counts to the least-loaded rank, ties to the
    // lower rank and entry), and the pairs (per head) this rank and all
    // ranks compute.
    std::vector<int32_t> entry_rank;
    double shard_pairs = 0, total_pairs = 0;
    int64_t shard_entries = 0;
    // Allowed (query, key) pairs of entry e, per head.
    double entry_pairs(const Entry &e) const;
    // With the environment variable CQSA_DEBUG set (not "0"), build() also
    // re-checks the plan by brute force (verify()); debug_checked says so.
    bool debug_checked = false;
    // Every allowed ordered block pair lies in exactly one entry; runs are
    // sorted, disjoint and in range; slots number each query block's
    // entries 0..n-1; the device work lists cover each entry's rows once.
    // Returns "" or what is violated.  Pair check up to 4096 blocks.
    std::string verify() const;

    // rows_per_unit: query rows one CTA covers; bn: key tile width.  With
    // spec.fused, one entry per query block holds the allowed key blocks of
    // all its tasks (the kernel's online softmax merges them) and writes the
    // output directly; otherwise one entry per (task, query block) with a
    // partial slot.
    WorkList device_worklist(int rows_per_unit, int bn, int heads) const;
    // This rank's part of a sharded forward: one entry per query block with
    // the union of the key runs of this rank's entries, flagged SEG_FIRST
    // only, so that the kernel leaves the rank's normalised partial and its
    // lse in the fp32 accumulator at the global row.
    WorkList partial_worklist(int rows_per_unit, int bn, int heads) const;
    // Key-stationary work list for the key and value gradients: one entry
    // per (task, key block) with the runs of query blocks the task's mask
    // allows (with spec.fused: one entry per key block over all tasks).
    // kv_slot of each entry numbers the tasks of a key block (partial slots);
    // *max_kv_slots gets the most any block has.
    WorkList device_worklist_kv(int rows_per_unit, int bn, int heads, int64_t *max_kv_slots) const;
    // The same two lists (partial slots, never fused) over only the entries
    // `use` selects, e.g. this rank's of a sharded plan: query-block slots
    // are renumbered among them, *nslots gets their count per block.
    WorkList device_worklist_sel(int rows_per_unit, int bn, int heads, const std::vector<char> &use,
                                 std::vector<int32_t> *nslots) const;
    WorkList device_worklist_kv_sel(int rows_per_unit, int bn, int heads, const std::vector<char> &use,
                                    int64_t *max_kv_slots) const;
    // Entries of this rank (all entries when the plan is not sharded).
    std::vector<char> shard_use() const;
    // Owner exchange of this rank (see ShardLayout); elem_bytes of the
    // gathered output rows.
    ShardLayout shard_layout(int elem_bytes) const;
    // Work list of leaf t reading Q, K, V from the block pools of `pool`.
    WorkList leaf_worklist(int64_t t, const PoolPlan &pool, int rows_per_unit, int bn, int heads) const;
    // Merge segments of leaf t in host mode (one per query block with an
    // entry), with first/last-touch flags in leaf order; the D2H copies of
    // finished rows follow them.
    std::vector<MergeSeg> leaf_merge_segments(int64_t t) const;
    // Members of leaf t whose Q (resp. K/V) rows a streamed task needs.
    void leaf_needs(int64_t t, std::vector<char> *need_q, std::vector<char> *need_kv) const;

private:
    // One entry per query block over the key blocks of the entries `use`
    // selects, as maximal runs.
    WorkList union_worklist(const std::vector<char> &use, int32_t flags, int rows_per_unit, int bn,
                            int heads) const;
    WorkList kv_worklist(int rows_per_unit, int bn, int heads, const std::vector<char> &use, bool fused,
                         int64_t *max_kv_slots) const;
    void assign_shards();

public:

    // Simulate the block cache with the given capacities; false if some
    // task (with its predecessor) needs more slots than there are.
    bool plan_pool(int64_t q_slots, int64_t kv_slots, PoolPlan *out) const;

    // Streamed backward: the block cache with `slots` slots (false if a task
    // and its predecessor need more), its device arena for head group g, and
    // the two work lists of leaf t in cache coordinates (rows of block b at
    // slot * block): query-stationary (dq, one entry per (task, query
    // block)) and key-stationary (dk and dv, one entry per (task, key
    // block)); each entry's sums go to the block's own slot rows.  With
    // grouped-query attention the key-stationary list's units are ordered
    // by query head modulo the group size (one launch per residue).
    bool plan_bwd_cache(int64_t slots, BwdCachePlan *out) const;
    size_t bwd_arena_bytes(int g, const BwdCachePlan &c) const;
    WorkList leaf_bwd_q_worklist(int64_t t, const BwdCachePlan &c, int rows_per_unit, int bn, int heads) const;
    WorkList leaf_bwd_kv_worklist(int64_t t, const BwdCachePlan &c, int rows_per_unit, int bn, int heads) const;
    BwdCachePlan bwd_cache;         // cache plan of the chosen backward sizing
    BwdSizing bwd_sizing;
    int64_t bwd_min_slots = 0, bwd_full_slots = 0;
    PoolPlan pool;                  // cache plan of the chosen sizing
    int64_t min_q_slots = 0, min_kv_slots = 0, full_q_slots = 0, full_kv_slots = 0;

    // Arena bytes of each mode for a head group g (host) / all heads (device).
    size_t host_arena_bytes(int g, const PoolPlan &pool) const;
    size_t device_arena_bytes() const;
    // The resident schedule (see HostLaunch): blocks per arrival group, the
    // launches, and its arena for a head group g.
    int64_t arrival_blocks() const;
    std::vector<HostLaunch> host_launches(int rows_per_unit, int bn, int heads) const;
    size_t resident_arena_bytes(int g, int sets, std::vector<HostLaunch> *launches) const;
    std::vector<HostLaunch> host_sched;  // the chosen resident schedule (empty: task by task)

private:
    // Bytes of leaf_worklist(t, pool, rows_per_unit, *, heads) and of the two
    // streamed-backward lists of leaf t, counted without building them (the
    // sizing loops try many caches): the same entries, the same runs after
    // joining rows that continue each other, and one unit per head and
    // chunk of an entry's rows that some key (query) of its runs reaches
    // under the causal rule.  verify() checks them against the built lists.
    size_t leaf_wl_bytes(int64_t t, const PoolPlan &pool, int rows_per_unit, int heads) const;
    size_t leaf_bwd_wl_bytes(int64_t t, const BwdCachePlan &c, int rows_per_unit, int heads) const;
    // What those counts need that does not depend on the cache, per leaf:
    // entries; units per head for chunks of 64, 128 and 256 rows; key
    // blocks over all entries (runs before joining), and for each member m
    // how many entries list the key blocks of members m and m + 1 one after
    // the other when those blocks are consecutive (a run joins there when
    // their slots are adjacent); the same for the key-stationary list (per
    // key member, its query members).
    struct LeafCount {
        int64_t ne_q = 0, nu_q[3] = {0, 0, 0}, keys_q = 0;
        std::vector<std::pair<int32_t, int32_t>> adj_q;
        int64_t ne_kv = 0, nu_kv[3] = {0, 0, 0}, qrys_kv = 0;
        std::vector<std::pair<int32_t, int32_t>> adj_kv;
    };
    std::vector<LeafCount> leaf_counts_;
    // Blocks each leaf task needs as Q and as K/V (forward), and touches
    // (backward), in member order: fixed by the plan, used by every cache
    // simulation of the sizing loops.
    std::vector<std::vector<int64_t>> need_q_, need_kv_, bwd_blocks_;
    void count_leaves();
    std::vector<int64_t> entry_begin_of_leaf_;  // first entry index of each leaf
    std::vector<int32_t> first_leaf_, last_leaf_; // per query block
    void size_plan();
    void size_bwd();
};

// Lexicographically first perfect difference set of size l mod l(l-1)+1
// containing {0, 1}; false if none exists.
bool find_difference_set(int l, std::vector<int> *D);

// Byte offsets of the sub-buffers of an arena, 256-byte aligned.
struct ArenaLayout {
    size_t total = 0;
    size_t take(size_t bytes) {
        size_t off = total;
        total += (bytes + 255) & ~size_t(255);
        return off;
    }
};

}  // namespace cqsa
