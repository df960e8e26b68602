// planner.cpp -- CQS planner (see planner.h for the sources it follows).
#include "planner.h"

#include <stdlib.h>

#include <algorithm>
#include <map>
#include <numeric>
#include <queue>
#include <unordered_map>

namespace cqsa {

// ---------------------------------------------------------------------------
// Perfect difference sets ("The CQS Divide"; arXiv abstract: cyclic quorum
// sets).  D of size l mod c = l(l-1)+1 such that every nonzero residue is a
// difference of two members exactly once.  Depth-first search in increasing
// order, so the first set found is the lexicographically first one that
// starts 0, 1.
// ---------------------------------------------------------------------------
static bool pds_search(int c, int l, std::vector<int> *cur, std::vector<char> *used) {
    if ((int)cur->size() == l) return true;
    for (int x = cur->back() + 1; x < c; ++x) {
        // Remaining slots must still fit below c.
        if (c - x < l - (int)cur->size()) break;
        std::vector<int> added;
        bool ok = true;
        for (int y : *cur) {
            const int a = ((x - y) % c + c) % c;
            const int b = (c - a) % c;
            if ((*used)[a] || (*used)[b] || a == b) { ok = false; break; }
            (*used)[a] = (*used)[b] = 1;
            added.push_back(a);
            added.push_back(b);
        }
        if (ok) {
            cur->push_back(x);
            if (pds_search(c, l, cur, used)) return true;
            cur->pop_back();
        }
        for (int a : added) (*used)[a] = 0;
    }
    return false;
}

bool find_difference_set(int l, std::vector<int> *D) {
    D->clear();
    if (l < 2 || l > 64) return false;
    const int c = l * (l - 1) + 1;
    std::vector<int> cur = {0, 1};
    std::vector<char> used(c, 0);
    used[1] = used[c - 1] = 1;
    if (l == 2) { *D = cur; return true; }
    if (!pds_search(c, l, &cur, &used)) return false;
    *D = cur;
    return true;
}

// ---------------------------------------------------------------------------
// Plan construction.
// ---------------------------------------------------------------------------
namespace {

struct Node {
    std::vector<int> path;
    std::vector<int64_t> blocks;
    std::vector<std::vector<int>> chunk;  // [level][member] chunk index at that level
};

}  // namespace

std::string Planner::build(const PlanSpec &s, int *code) {
    spec = s;
    *code = 1;  // INVALID_ARG unless changed
    if (s.N <= 0 || s.H <= 0 || s.d <= 0) return "N, H and d must be positive";
    if (s.levels < 1 || s.levels > kMaxLevels) return "levels must be in 1..4";
    // Rows are 32-bit in the work lists and kernels, which add a tile or
    // unit width (at most 256) to a row: keep that below 2^31.
    if (s.N > (int64_t)kMaxN) return "N must be at most 2^31 - 4096";
    if (s.Hkv < 0 || (s.Hkv > 0 && s.H % s.Hkv != 0))
        return "the query heads must be a multiple of the key/value heads";
    if (spec.Hkv == 0) spec.Hkv = s.H;
    if (s.B < 1) return "the batch B must be at least 1";
    if (s.shard_count < 1 || s.shard_rank < 0 || s.shard_rank >= s.shard_count)
        return "the shard rank must be in 0..shard_count-1 (shard_count >= 1)";
    levels.clear();
    num_blocks = 1;
    for (int i = 0; i < s.levels; ++i) {
        Level L;
        L.l = s.l[i];
        if (L.l < 2 || L.l > 16) return "each level's l must be in 2..16";
        L.c = L.l * (L.l - 1) + 1;
        if (!find_difference_set(L.l, &L.D)) {
            *code = 2;
            return "no perfect difference set of size " + std::to_string(L.l) + " mod " +
                   std::to_string(L.c);
        }
        num_blocks *= L.c;
        levels.push_back(L);
    }
    // N need not be a multiple of the block count: blocks of ceil(N / P)
    // tokens, and positions at or past N belong to no pair.
    block = (s.N + num_blocks - 1) / num_blocks;

    // Recursive division ("The Recursive Benefit"): level i divides each
    // parent's token sequence (its blocks in increasing order) into c_i equal
    // chunks and forms the c_i subsequences {(x + k) mod c_i : x in D_i}.
    std::vector<Node> frontier(1);
    frontier[0].blocks.resize(num_blocks);
    std::iota(frontier[0].blocks.begin(), frontier[0].blocks.end(), 0);
    for (int i = 0; i < s.levels; ++i) {
        const Level &L = levels[i];
        std::vector<Node> next;
        next.reserve(frontier.size() * L.c);
        for (const Node &p : frontier) {
            const int64_t n = (int64_t)p.blocks.size();
            const int64_t per = n / L.c;
            for (int k = 0; k < L.c; ++k) {
                std::vector<char> in(L.c, 0);
                for (int x : L.D) in[(x + k) % L.c] = 1;
                Node ch;
                ch.path = p.path;
                ch.path.push_back(k);
                ch.chunk.resize(i + 1);
                for (int64_t m = 0; m < n; ++m) {
                    const int a = (int)(m / per);
                    if (!in[a]) continue;
                    ch.blocks.push_back(p.blocks[m]);
                    for (int j = 0; j < i; ++j) ch.chunk[j].push_back(p.chunk[j][m]);
                    ch.chunk[i].push_back(a);
                }
                next.push_back(std::move(ch));
            }
        }
        frontier.swap(next);
    }

    // CQS mask of a leaf ("Implementation"): at every level, a pair of
    // distinct chunks is allowed; the diagonal pair (a, a) only in the
    // subsequence that owns it, k = (a - D[0]) mod c.  Causal keeps key
    // blocks at or before the query block (the diagonal block's upper
    // triangle is removed inside the kernel).
    leaves.clear();
    entries.clear();
    entry_begin_of_leaf_.clear();
    slots_per_block.assign(num_blocks, 0);
    first_leaf_.assign(num_blocks, -1);
    last_leaf_.assign(num_blocks, -1);
    max_task_rows = 0;
    for (int64_t t = 0; t < (int64_t)frontier.size(); ++t) {
        const Node &nd = frontier[t];
        const int64_t n = (int64_t)nd.blocks.size();
        max_task_rows = std::max<int64_t>(max_task_rows, n * block);
        entry_begin_of_leaf_.push_back((int64_t)entries.size());
        for (int64_t mq = 0; mq < n; ++mq) {
            if (block_rows(nd.blocks[mq]) == 0) continue;  // no query row in this block
            Entry e;
            e.task = t;
            e.qb = nd.blocks[mq];
            e.mq = (int32_t)mq;
            for (int64_t mk = 0; mk < n; ++mk) {
                bool ok = true;
                for (int i = 0; i < s.levels && ok; ++i) {
                    const Level &L = levels[i];
                    const int a = nd.chunk[i][mq], b = nd.chunk[i][mk];
                    if (a == b) {
                        const int owner = ((a - L.D[0]) % L.c + L.c) % L.c;
                        ok = (owner == nd.path[i]);
                    }
                }
                if (ok && s.causal && nd.blocks[mk] > nd.blocks[mq]) ok = false;
                if (ok && block_rows(nd.blocks[mk]) == 0) ok = false;
                if (!ok) continue;
                const int64_t kb = nd.blocks[mk];
                if (!e.runs.empty() && e.runs.back().b1 + 1 == kb &&
                    e.runs.back().m0 + (e.runs.back().b1 - e.runs.back().b0) + 1 == mk) {
                    e.runs.back().b1 = kb;
                } else {
                    e.runs.push_back(KeyRun{kb, kb, (int32_t)mk});
                }
            }
            if (e.runs.empty()) continue;
            e.slot = slots_per_block[e.qb]++;
            if (first_leaf_[e.qb] < 0) first_leaf_[e.qb] = (int32_t)t;
            last_leaf_[e.qb] = (int32_t)t;
            entries.push_back(std::move(e));
        }
        Leaf lf;
        lf.path = nd.path;
        lf.blocks = nd.blocks;
        leaves.push_back(std::move(lf));
    }
    entry_begin_of_leaf_.push_back((int64_t)entries.size());
    max_slots = 0;
    for (int32_t v : slots_per_block) max_slots = std::max<int64_t>(max_slots, v);
    assign_shards();
    count_leaves();
    size_plan();
    size_bwd();
    const char *dbg = getenv("CQSA_DEBUG");
    if (dbg && dbg[0] && !(dbg[0] == '0' && dbg[1] == 0)) {
        const std::string bad = verify();
        if (!bad.empty()) {
            *code = 9;  // CQSA_ERR_INTERNAL
            return "CQSA_DEBUG: plan invariant violated: " + bad;
        }
        debug_checked = true;
    }
    *code = 0;
    return "";
}

static size_t wl_bytes(const WorkList &wl);

std::string Planner::verify() const {
    const int64_t P = num_blocks;
    // Runs: sorted, disjoint, in range; slots: 0..n-1 per query block.
    std::vector<int32_t> seen_slots(P, 0);
    for (const Entry &e : entries) {
        if (e.qb < 0 || e.qb >= P) return "query block out of range";
        int64_t prev = -1;
        for (const KeyRun &r : e.runs) {
            if (r.b0 > r.b1 || r.b0 <= prev || r.b1 >= P) return "key runs not sorted, disjoint and in range";
            prev = r.b1;
        }
        if (e.slot != seen_slots[e.qb]++) return "slots do not number a query block's entries in order";
    }
    for (int64_t b = 0; b < P; ++b)
        if (seen_slots[b] != slots_per_block[b]) return "slot count mismatch";
    // The counted work-list sizes of the sizing loops equal the built lists'.
    if (sizing.head_group > 0 && !sizing.resident)
        for (int64_t t = 0; t < (int64_t)leaves.size(); ++t) {
            const int rpu = unit_rows_for(spec.elem_bytes);
            if (leaf_wl_bytes(t, pool, rpu, sizing.head_group) !=
                wl_bytes(leaf_worklist(t, pool, rpu, key_tile_for(spec.elem_bytes), sizing.head_group)))
                return "counted streamed work-list size differs from the built list";
        }
    if (bwd_sizing.head_group > 0)
        for (int64_t t = 0; t < (int64_t)leaves.size(); ++t) {
            const int tile = spec.elem_bytes == 2 ? 128 : 64, g = bwd_sizing.head_group;
            if (leaf_bwd_wl_bytes(t, bwd_cache, tile, g) !=
                wl_bytes(leaf_bwd_q_worklist(t, bwd_cache, tile, tile, g)) +
                    wl_bytes(leaf_bwd_kv_worklist(t, bwd_cache, tile, tile, g)))
                return "counted backward work-list size differs from the built lists";
        }
    // Exactly-once coverage of the allowed block pairs.
    if (P <= 4096) {
        std::vector<uint8_t> hits((size_t)P * P, 0);
        for (const Entry &e : entries)
            for (const KeyRun &r : e.runs)
                for (int64_t kb = r.b0; kb <= r.b1; ++kb) {
                    uint8_t &h = hits[(size_t)e.qb * P + kb];
                    if (h == 255) return "pair counted 255 times";
                    ++h;
                }
        for (int64_t qb = 0; qb < P; ++qb)
            for (int64_t kb = 0; kb < P; ++kb) {
                const bool allowed = block_rows(qb) > 0 && block_rows(kb) > 0 && (!spec.causal || kb <= qb);
                if (hits[(size_t)qb * P + kb] != (allowed ? 1 : 0)) return "a block pair is not covered exactly once";
            }
    }
    // Device work list: the units of each entry cover its rows once per head.
    const int rows = unit_rows_for(spec.elem_bytes);
    WorkList wl = device_worklist(rows, key_tile_for(spec.elem_bytes), spec.H);
    std::vector<int64_t> covered(wl.entries.size(), 0);
    for (const WlUnit &u : wl.units) {
        if (u.entry < 0 || u.entry >= (int32_t)wl.entries.size()) return "unit entry out of range";
        const WlEntry &e = wl.entries[u.entry];
        if (u.q0 < e.q_lo || u.q0 >= e.q_hi || u.head < 0 || u.head >= spec.H) return "unit outside its entry";
        covered[u.entry] += std::min<int64_t>(rows, e.q_hi - u.q0);
    }
    for (size_t i = 0; i < wl.entries.size(); ++i)
        if (covered[i] != (int64_t)(wl.entries[i].q_hi - wl.entries[i].q_lo) * spec.H)
            return "device units do not cover an entry's rows once per head";
    return "";
}

// ---------------------------------------------------------------------------
// Work lists.
// ---------------------------------------------------------------------------
// group[ei]: the task of entry ei (units of one task and head read the same
// key and value blocks).
static void add_units(WorkList *wl, int heads, int rows_per_unit, int bn, int causal,
                      const std::vector<int64_t> &group) {
    std::vector<WlUnit> u;
    for (int32_t ei = 0; ei < (int32_t)wl->entries.size(); ++ei) {
        const WlEntry &e = wl->entries[ei];
        for (int h = 0; h < heads; ++h)
            for (int64_t q0 = e.q_lo; q0 < e.q_hi; q0 += rows_per_unit) {
                WlUnit x;
                x.entry = ei;
                x.q0 = (int32_t)q0;  // < N <= kMaxN
                x.head = h;
                x.ntiles = unit_key_tiles(e, wl->runs.data(), x.q0, rows_per_unit, causal, bn);
                if (x.ntiles > 0) u.push_back(x);
            }
    }
    // Longest units first, in classes of 32 key tiles (coarse LPT order, so
    // the tail of the grid is short), and inside a class by head, then task:
    // the CTAs in flight at one time then share a few tasks' key and value
    // blocks of one head, which stay in L2 instead of being fetched again
    // from HBM for every (entry, head).
    std::stable_sort(u.begin(), u.end(), [&](const WlUnit &a, const WlUnit &b) {
        const int ca = a.ntiles / 32, cb = b.ntiles / 32;
        if (ca != cb) return ca > cb;
        if (a.head != b.head) return a.head < b.head;
        return group[a.entry] < group[b.entry];
    });
    wl->units.swap(u);
}

double Planner::entry_pairs(const Entry &e) const {
    const double qr = (double)block_rows(e.qb);
    double n = 0;
    for (const KeyRun &r : e.runs)
        for (int64_t b = r.b0; b <= r.b1; ++b)
            n += (spec.causal && b == e.qb) ? qr * (qr + 1) / 2 : qr * (double)block_rows(b);
    return n;
}

void Planner::assign_shards() {
    const int G = std::max(1, spec.shard_count);
    entry_rank.assign(entries.size(), 0);
    std::vector<double> cost(entries.size());
    total_pairs = 0;
    for (size_t i = 0; i < entries.size(); ++i) {
        cost[i] = entry_pairs(entries[i]);
        total_pairs += cost[i];
    }
    if (G > 1) {
        std::vector<size_t> order(entries.size());
        for (size_t i = 0; i < order.size(); ++i) order[i] = i;
        std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) { return cost[a] > cost[b]; });
        std::vector<double> load(G, 0.0);
        for (size_t i : order) {
            int r = 0;
            for (int x = 1; x < G; ++x)
                if (load[x] < load[r]) r = x;
            entry_rank[i] = r;
            load[r] += cost[i];
        }
    }
    shard_pairs = 0;
    shard_entries = 0;
    for (size_t i = 0; i < entries.size(); ++i)
        if (entry_rank[i] == spec.shard_rank) {
            shard_pairs += cost[i];
            ++shard_entries;
        }
}

WorkList Planner::union_worklist(const std::vector<char> &use, int32_t flags, int rows_per_unit, int bn,
                                 int heads) const {
    // The tasks of a query block own disjoint sets of its allowed key
    // blocks; their union, as maximal runs, is one entry.
    WorkList wl;
    std::vector<int64_t> group;
    std::vector<std::vector<int64_t>> keys(num_blocks);
    for (size_t i = 0; i < entries.size(); ++i) {
        if (!use[i]) continue;
        const Entry &e = entries[i];
        for (const KeyRun &r : e.runs)
            for (int64_t b = r.b0; b <= r.b1; ++b) keys[e.qb].push_back(b);
    }
    for (int64_t qb = 0; qb < num_blocks; ++qb) {
        std::vector<int64_t> &kb = keys[qb];
        if (kb.empty()) continue;
        std::sort(kb.begin(), kb.end());
        WlEntry w{};
        w.q_lo = (int32_t)(qb * block);
        w.q_hi = (int32_t)block_end(qb);
        w.out_lo = w.q_lo;
        w.flags = flags;
        w.run_begin = (int32_t)wl.runs.size();
        for (size_t i = 0; i < kb.size(); ++i) {
            if (i > 0 && kb[i] == kb[i - 1] + 1) {
                wl.runs.back().k_hi = (int32_t)block_end(kb[i]);
            } else {
                WlRun x{};
                x.k_lo = (int32_t)(kb[i] * block);
                x.k_hi = (int32_t)block_end(kb[i]);
                wl.runs.push_back(x);
            }
        }
        w.run_count = (int32_t)wl.runs.size() - w.run_begin;
        wl.entries.push_back(w);
        group.push_back(0);
    }
    add_units(&wl, heads, rows_per_unit, bn, spec.causal, group);
    return wl;
}

WorkList Planner::partial_worklist(int rows_per_unit, int bn, int heads) const {
    std::vector<char> use(entries.size());
    for (size_t i = 0; i < entries.size(); ++i) use[i] = entry_rank[i] == spec.shard_rank;
    return union_worklist(use, SEG_FIRST, rows_per_unit, bn, heads);
}

WorkList Planner::device_worklist(int rows_per_unit, int bn, int heads) const {
    WorkList wl;
    std::vector<int64_t> group;
    if (spec.fused) return union_worklist(std::vector<char>(entries.size(), 1), SEG_FIRST | SEG_LAST,
                                          rows_per_unit, bn, heads);
    for (const Entry &e : entries) {
        group.push_back(e.task);
        WlEntry w{};
        w.q_lo = (int32_t)(e.qb * block);
        w.q_hi = (int32_t)block_end(e.qb);
        w.q_goff = 0;
        w.slot = (int32_t)e.slot;
        w.out_lo = w.q_lo;
        w.run_begin = (int32_t)wl.runs.size();
        w.run_count = (int32_t)e.runs.size();
        for (const KeyRun &r : e.runs) {
            WlRun x{};
            x.k_lo = (int32_t)(r.b0 * block);
            x.k_hi = (int32_t)block_end(r.b1);
            x.k_goff = 0;
            wl.runs.push_back(x);
        }
        wl.entries.push_back(w);
    }
    add_units(&wl, heads, rows_per_unit, bn, spec.causal, group);
    return wl;
}

std::vector<char> Planner::shard_use() const {
    std::vector<char> use(entries.size());
    for (size_t i = 0; i < entries.size(); ++i) use[i] = entry_rank[i] == spec.shard_rank;
    return use;
}

WorkList Planner::device_worklist_kv(int rows_per_unit, int bn, int heads, int64_t *max_kv_slots) const {
    return kv_worklist(rows_per_unit, bn, heads, std::vector<char>(entries.size(), 1), spec.fused != 0,
                       max_kv_slots);
}

WorkList Planner::device_worklist_kv_sel(int rows_per_unit, int bn, int heads, const std::vector<char> &use,
                                         int64_t *max_kv_slots) const {
    return kv_worklist(rows_per_unit, bn, heads, use, false, max_kv_slots);
}

WorkList Planner::device_worklist_sel(int rows_per_unit, int bn, int heads, const std::vector<char> &use,
                                      std::vector<int32_t> *nslots) const {
    WorkList wl;
    std::vector<int64_t> group;
    nslots->assign(num_blocks, 0);
    for (size_t i = 0; i < entries.size(); ++i) {
        if (!use[i]) continue;
        const Entry &e = entries[i];
        group.push_back(e.task);
        WlEntry w{};
        w.q_lo = (int32_t)(e.qb * block);
        w.q_hi = (int32_t)block_end(e.qb);
        w.slot = (*nslots)[e.qb]++;
        w.out_lo = w.q_lo;
        w.run_begin = (int32_t)wl.runs.size();
        w.run_count = (int32_t)e.runs.size();
        for (const KeyRun &r : e.runs) {
            WlRun x{};
            x.k_lo = (int32_t)(r.b0 * block);
            x.k_hi = (int32_t)block_end(r.b1);
            wl.runs.push_back(x);
        }
        wl.entries.push_back(w);
    }
    add_units(&wl, heads, rows_per_unit, bn, spec.causal, group);
    return wl;
}

WorkList Planner::kv_worklist(int rows_per_unit, int bn, int heads, const std::vector<char> &use, bool fused,
                              int64_t *max_kv_slots) const {
    // kb -> (task, query blocks) in task order; pairs come from the forward
    // entries, whose key runs already carry every level's CQS mask.
    std::vector<std::vector<std::pair<int64_t, std::vector<int64_t>>>> by_kb(num_blocks);
    for (size_t i = 0; i < entries.size(); ++i) {
        if (!use[i]) continue;
        const Entry &e = entries[i];
        for (const KeyRun &r : e.runs)
            for (int64_t kb = r.b0; kb <= r.b1; ++kb) {
                auto &lst = by_kb[kb];
                if (fused) {
                    if (lst.empty()) lst.push_back({0, {}});
                    lst.back().second.push_back(e.qb);
                } else {
                    if (lst.empty() || lst.back().first != e.task) lst.push_back({e.task, {}});
                    lst.back().second.push_back(e.qb);
                }
            }
    }
    WorkList wl;
    std::vector<int64_t> group;
    *max_kv_slots = 0;
    for (int64_t kb = 0; kb < num_blocks; ++kb) {
        int32_t slot = 0;
        for (auto &tq : by_kb[kb]) {
            std::vector<int64_t> &qs = tq.second;
            std::sort(qs.begin(), qs.end());
            WlEntry w{};
            w.q_lo = (int32_t)(kb * block);
            w.q_hi = (int32_t)block_end(kb);
            w.slot = slot++;
            w.out_lo = w.q_lo;
            w.flags = fused ? (SEG_FIRST | SEG_LAST) : 0;
            w.run_begin = (int32_t)wl.runs.size();
            for (size_t i = 0; i < qs.size(); ++i) {
                if (i > 0 && qs[i] == qs[i - 1] + 1) {
                    wl.runs.back().k_hi = (int32_t)block_end(qs[i]);
                } else {
                    WlRun x{};
                    x.k_lo = (int32_t)(qs[i] * block);
                    x.k_hi = (int32_t)block_end(qs[i]);
                    wl.runs.push_back(x);
                }
            }
            w.run_count = (int32_t)wl.runs.size() - w.run_begin;
            wl.entries.push_back(w);
            group.push_back(tq.first);
        }
        *max_kv_slots = std::max<int64_t>(*max_kv_slots, slot);
    }
    std::vector<WlUnit> u;
    for (int32_t ei = 0; ei < (int32_t)wl.entries.size(); ++ei) {
        const WlEntry &e = wl.entries[ei];
        for (int h = 0; h < heads; ++h)
            for (int64_t k0 = e.q_lo; k0 < e.q_hi; k0 += rows_per_unit) {
                const int32_t r0 = (int32_t)k0;  // < N <= kMaxN
                WlUnit x{ei, r0, h, unit_query_tiles(e, wl.runs.data(), r0, spec.causal, bn)};
                if (x.ntiles > 0) u.push_back(x);
            }
    }
    std::stable_sort(u.begin(), u.end(), [&](const WlUnit &a, const WlUnit &b) {
        const int ca = a.ntiles / 32, cb = b.ntiles / 32;
        if (ca != cb) return ca > cb;
        if (a.head != b.head) return a.head < b.head;
        return group[a.entry] < group[b.entry];
    });
    wl.units.swap(u);
    return wl;
}

WorkList Planner::leaf_worklist(int64_t t, const PoolPlan &pool, int rows_per_unit, int bn, int heads) const {
    // Q rows come from Q slot q_slot * block, K and V rows from KV slot
    // kv_slot * block; partial outputs go to the task's local rows mq * block.
    WorkList wl;
    for (int64_t i = entry_begin_of_leaf_[t]; i < entry_begin_of_leaf_[t + 1]; ++i) {
        const Entry &e = entries[i];
        const int64_t qs = pool.q_slot[t][e.mq];
        WlEntry w{};
        w.q_lo = (int32_t)(qs * block);
        w.q_hi = (int32_t)(qs * block + block_rows(e.qb));
        w.q_goff = (int32_t)((e.qb - qs) * block);
        w.slot = 0;
        w.out_lo = (int32_t)(e.mq * block);
        w.flags = (first_leaf_[e.qb] == t ? SEG_FIRST : 0) | (last_leaf_[e.qb] == t ? SEG_LAST : 0);
        w.run_begin = (int32_t)wl.runs.size();
        for (const KeyRun &r : e.runs) {
            for (int64_t kb = r.b0; kb <= r.b1; ++kb) {
                const int64_t ks = pool.kv_slot[t][r.m0 + (kb - r.b0)];
                const int32_t lo = (int32_t)(ks * block), goff = (int32_t)((kb - ks) * block);
                if ((int32_t)wl.runs.size() > w.run_begin && wl.runs.back().k_hi == lo &&
                    wl.runs.back().k_goff == goff) {
                    // Contiguous slots: one run.  A partial last block ends its
                    // run short, so nothing is ever appended past it.
                    wl.runs.back().k_hi = lo + (int32_t)block_rows(kb);
                } else {
                    WlRun x{};
                    x.k_lo = lo;
                    x.k_hi = lo + (int32_t)block_rows(kb);
                    x.k_goff = goff;
                    wl.runs.push_back(x);
                }
            }
        }
        w.run_count = (int32_t)wl.runs.size() - w.run_begin;
        wl.entries.push_back(w);
    }
    add_units(&wl, heads, rows_per_unit, bn, spec.causal, std::vector<int64_t>(wl.entries.size(), t));
    return wl;
}

std::vector<MergeSeg> Planner::leaf_merge_segments(int64_t t) const {
    std::vector<MergeSeg> segs;
    for (int64_t i = entry_begin_of_leaf_[t]; i < entry_begin_of_leaf_[t + 1]; ++i) {
        const Entry &e = entries[i];
        MergeSeg s{};
        s.local_lo = (int32_t)(e.mq * block);
        s.rows = (int32_t)block_rows(e.qb);
        s.global_lo = (int32_t)(e.qb * block);
        s.flags = (first_leaf_[e.qb] == t ? SEG_FIRST : 0) | (last_leaf_[e.qb] == t ? SEG_LAST : 0);
        segs.push_back(s);
    }
    return segs;
}

void Planner::leaf_needs(int64_t t, std::vector<char> *need_q, std::vector<char> *need_kv) const {
    const size_t n = leaves[t].blocks.size();
    need_q->assign(n, 0);
    need_kv->assign(n, 0);
    for (int64_t i = entry_begin_of_leaf_[t]; i < entry_begin_of_leaf_[t + 1]; ++i) {
        const Entry &e = entries[i];
        (*need_q)[e.mq] = 1;
        for (const KeyRun &r : e.runs)
            for (int64_t b = r.b0; b <= r.b1; ++b) (*need_kv)[r.m0 + (b - r.b0)] = 1;
    }
}

// ---------------------------------------------------------------------------
// Block cache of the streamed path (Belady; see planner.h).
// ---------------------------------------------------------------------------
namespace {

// Blocks each leaf task needs as Q and as K/V, in member order.
void task_needs(const Planner &pl, std::vector<std::vector<int64_t>> *nq, std::vector<std::vector<int64_t>> *nkv) {
    const size_t T = pl.leaves.size();
    nq->assign(T, {});
    nkv->assign(T, {});
    std::vector<char> q, kv;
    for (size_t t = 0; t < T; ++t) {
        pl.leaf_needs((int64_t)t, &q, &kv);
        for (size_t m = 0; m < q.size(); ++m) {
            if (q[m]) (*nq)[t].push_back(pl.leaves[t].blocks[m]);
            if (kv[m]) (*nkv)[t].push_back(pl.leaves[t].blocks[m]);
        }
    }
}

// One cache of `cap` slots over the task sequence; fills slot_of[t][block]
// and the copies.  False when a task and its predecessor need more than cap.
// A miss takes the lowest slot never used, else evicts, among the slots
// whose block neither this task nor the previous one needs, the block used
// again farthest ahead (the lowest slot on a tie).  The candidates sit in a
// max-heap keyed by (next use, -slot), kept lazily: an entry counts only
// while its slot still holds a block with that key and is unprotected; a
// protected slot rejoins the heap when its protection ends.
bool simulate(const std::vector<std::vector<int64_t>> &need, int64_t cap, int kind,
              std::vector<std::unordered_map<int64_t, int32_t>> *slot_of, std::vector<std::vector<PoolCopy>> *copies,
              int64_t *ncopies) {
    const size_t T = need.size();
    std::unordered_map<int64_t, std::vector<int64_t>> uses;  // block -> tasks using it, increasing
    for (size_t t = 0; t < T; ++t)
        for (int64_t b : need[t]) {
            std::vector<int64_t> &u = uses[b];
            if (u.empty() || u.back() != (int64_t)t) u.push_back((int64_t)t);
        }
    auto next_use = [&](int64_t b, int64_t t) -> int64_t {
        const std::vector<int64_t> &u = uses[b];
        auto it = std::upper_bound(u.begin(), u.end(), t);
        return it == u.end() ? INT64_MAX : *it;
    };
    std::vector<int64_t> slot_block(cap, -1), key(cap, -1), guard(cap, -1);  // guard: protected through this task
    std::unordered_map<int64_t, int32_t> where;
    std::priority_queue<std::pair<int64_t, int64_t>> heap;  // (next use, -slot)
    std::vector<std::vector<int32_t>> rejoin(T + 2);       // slots whose protection ends before task t
    int64_t next_free = 0;
    slot_of->assign(T, {});
    auto protect = [&](int32_t sl, int64_t b, int64_t t) {
        guard[sl] = t + 1;  // needed by task t: protected in tasks t and t + 1
        key[sl] = next_use(b, t);
        rejoin[t + 2].push_back(sl);
    };
    for (size_t t = 0; t < T; ++t) {
        for (int32_t sl : rejoin[t])
            if (slot_block[sl] >= 0 && guard[sl] == (int64_t)t - 1) heap.push({key[sl], -(int64_t)sl});
        for (int64_t b : need[t]) {
            auto hit = where.find(b);
            if (hit != where.end()) protect(hit->second, b, (int64_t)t);
        }
        for (int64_t b : need[t]) {
            auto hit = where.find(b);
            if (hit == where.end()) {
                int32_t slot = -1;
                if (next_free < cap) {
                    slot = (int32_t)next_free++;
                } else {
                    while (!heap.empty()) {
                        const std::pair<int64_t, int64_t> top = heap.top();
                        heap.pop();
                        const int32_t sl = (int32_t)(-top.second);
                        if (slot_block[sl] >= 0 && key[sl] == top.first && guard[sl] < (int64_t)t) {
                            slot = sl;
                            break;
                        }
                    }
                    if (slot < 0) return false;
                    where.erase(slot_block[slot]);
                }
                slot_block[slot] = b;
                where[b] = slot;
                protect(slot, b, (int64_t)t);
                (*copies)[t].push_back(PoolCopy{kind, b, slot});
                ++*ncopies;
                hit = where.find(b);
            }
            (*slot_of)[t][b] = hit->second;
        }
    }
    return true;
}

}  // namespace

bool Planner::plan_pool(int64_t q_slots, int64_t kv_slots, PoolPlan *out) const {
    const std::vector<std::vector<int64_t>> &nq = need_q_, &nkv = need_kv_;
    PoolPlan pp;
    pp.q_slots = q_slots;
    pp.kv_slots = kv_slots;
    const size_t T = leaves.size();
    pp.copies.assign(T, {});
    std::vector<std::unordered_map<int64_t, int32_t>> sq, skv;
    if (!simulate(nq, q_slots, 0, &sq, &pp.copies, &pp.q_copies)) return false;
    // K/V copies after the task's Q copies (one list per task).
    std::vector<std::vector<PoolCopy>> kvc(T);
    if (!simulate(nkv, kv_slots, 1, &skv, &kvc, &pp.kv_copies)) return false;
    pp.q_slot.assign(T, {});
    pp.kv_slot.assign(T, {});
    for (size_t t = 0; t < T; ++t) {
        pp.copies[t].insert(pp.copies[t].end(), kvc[t].begin(), kvc[t].end());
        const size_t n = leaves[t].blocks.size();
        pp.q_slot[t].assign(n, -1);
        pp.kv_slot[t].assign(n, -1);
        for (size_t m = 0; m < n; ++m) {
            const int64_t b = leaves[t].blocks[m];
            auto a = sq[t].find(b);
            if (a != sq[t].end()) pp.q_slot[t][m] = a->second;
            auto k = skv[t].find(b);
            if (k != skv[t].end()) pp.kv_slot[t][m] = k->second;
        }
    }
    *out = std::move(pp);
    return true;
}

// ---------------------------------------------------------------------------
// Memory sizing (layerthelatestinalattice.com summary: subproblems fit a
// stated memory budget).  Every byte the library holds on the device lives
// in one arena whose layout the runtime rebuilds with the same ArenaLayout
// steps, so these totals are exact.
// ---------------------------------------------------------------------------
static size_t wl_bytes(const WorkList &wl) {
    ArenaLayout a;
    a.take(wl.entries.size() * sizeof(WlEntry));
    a.take(wl.runs.size() * sizeof(WlRun));
    a.take(wl.units.size() * sizeof(WlUnit));
    return a.total;
}

size_t Planner::device_arena_bytes() const {
    const int64_t N = spec.N;
    ArenaLayout a;
    a.take(256);                                                        // error word
    if (!spec.fused) {
        a.take((size_t)max_slots * N * spec.H * spec.d * sizeof(float)); // partial O
        a.take((size_t)max_slots * spec.H * N * sizeof(float));          // partial lse
        a.take((size_t)num_blocks * sizeof(int32_t));                    // slots per block
    }
    WorkList wl = device_worklist(unit_rows_for(spec.elem_bytes), key_tile_for(spec.elem_bytes), spec.H);
    a.take(wl_bytes(wl));
    return a.total;
}

namespace {
size_t wl_sizes(size_t entries, size_t runs, size_t units) {
    ArenaLayout a;
    a.take(entries * sizeof(WlEntry));
    a.take(runs * sizeof(WlRun));
    a.take(units * sizeof(WlUnit));
    return a.total;
}

// Runs left after joining rows that continue the previous run (the rule of
// leaf_worklist and push_run): rows [lo, lo + n) with offset goff.
struct RunCount {
    size_t n = 0;
    bool have = false;
    int64_t hi = 0, goff = 0;
    void add(int64_t lo, int64_t rows, int64_t g) {
        if (!(have && hi == lo && goff == g)) {
            ++n;
            have = true;
            goff = g;
        }
        hi = lo + rows;
    }
};
}  // namespace

namespace {
std::vector<std::vector<int64_t>> bwd_task_blocks(const Planner &pl);
}  // namespace

void Planner::count_leaves() {
    task_needs(*this, &need_q_, &need_kv_);
    bwd_blocks_ = bwd_task_blocks(*this);
    const int rpus[3] = {64, 128, 256};
    leaf_counts_.assign(leaves.size(), LeafCount{});
    for (int64_t t = 0; t < (int64_t)leaves.size(); ++t) {
        LeafCount &c = leaf_counts_[t];
        const size_t n = leaves[t].blocks.size();
        std::vector<int32_t> adj_q(n, 0), adj_kv(n, 0);
        std::vector<std::vector<int32_t>> qs_of(n);
        for (int64_t i = entry_begin_of_leaf_[t]; i < entry_begin_of_leaf_[t + 1]; ++i) {
            const Entry &e = entries[i];
            ++c.ne_q;
            for (const KeyRun &r : e.runs) {
                c.keys_q += r.b1 - r.b0 + 1;
                for (int64_t kb = r.b0; kb < r.b1; ++kb) ++adj_q[r.m0 + (kb - r.b0)];
                for (int64_t kb = r.b0; kb <= r.b1; ++kb) qs_of[r.m0 + (kb - r.b0)].push_back(e.mq);
            }
            // A chunk is a unit when the entry's first key is at or before its last query.
            const int64_t q_lo = e.qb * block, q_hi = q_lo + block_rows(e.qb), k_first = e.runs.front().b0 * block;
            for (int x = 0; x < 3; ++x)
                for (int64_t q0 = q_lo; q0 < q_hi; q0 += rpus[x])
                    if (!spec.causal || k_first <= std::min<int64_t>(q0 + rpus[x], q_hi) - 1) ++c.nu_q[x];
        }
        for (size_t mk = 0; mk < n; ++mk) {
            std::vector<int32_t> &qm = qs_of[mk];
            if (qm.empty()) continue;
            std::sort(qm.begin(), qm.end());
            ++c.ne_kv;
            c.qrys_kv += (int64_t)qm.size();
            int64_t q_end = 0;  // one past the last query row (global)
            for (size_t j = 0; j < qm.size(); ++j) {
                const int64_t qb = leaves[t].blocks[qm[j]];
                q_end = std::max<int64_t>(q_end, qb * block + block_rows(qb));
                // Consecutive members with consecutive blocks (members need not hold consecutive blocks).
                if (j > 0 && qm[j] == qm[j - 1] + 1 && qb == leaves[t].blocks[qm[j - 1]] + 1) ++adj_kv[qm[j - 1]];
            }
            // A chunk of keys is a unit when some query is at or after its first key.
            const int64_t kb = leaves[t].blocks[mk], k_lo = kb * block, k_hi = k_lo + block_rows(kb);
            for (int x = 0; x < 3; ++x)
                for (int64_t k0 = k_lo; k0 < k_hi; k0 += rpus[x])
                    if (!spec.causal || q_end > k0) ++c.nu_kv[x];
        }
        for (size_t m = 0; m < n; ++m) {
            if (adj_q[m]) c.adj_q.push_back({(int32_t)m, adj_q[m]});
            if (adj_kv[m]) c.adj_kv.push_back({(int32_t)m, adj_kv[m]});
        }
    }
}

namespace {
int rpu_index(int rows) { return rows == 64 ? 0 : rows == 128 ? 1 : 2; }
}  // namespace

size_t Planner::leaf_wl_bytes(int64_t t, const PoolPlan &pool, int rows_per_unit, int heads) const {
    const LeafCount &c = leaf_counts_[t];
    // Members m and m + 1 listed here hold consecutive blocks; a run
    // continues across them when their slots are adjacent and block m is full.
    int64_t joins = 0;
    for (const auto &a : c.adj_q) {
        const int32_t m = a.first;
        if (pool.kv_slot[t][m + 1] == pool.kv_slot[t][m] + 1 && block_rows(leaves[t].blocks[m]) == block)
            joins += a.second;
    }
    return wl_sizes((size_t)c.ne_q, (size_t)(c.keys_q - joins), (size_t)c.nu_q[rpu_index(rows_per_unit)] * heads);
}

size_t Planner::leaf_bwd_wl_bytes(int64_t t, const BwdCachePlan &cp, int rows_per_unit, int heads) const {
    const LeafCount &c = leaf_counts_[t];
    const std::vector<int32_t> &ms = cp.member_slot[t];
    auto joined = [&](const std::vector<std::pair<int32_t, int32_t>> &adj) {
        int64_t j = 0;
        for (const auto &a : adj)
            if (ms[a.first + 1] == ms[a.first] + 1 && block_rows(leaves[t].blocks[a.first]) == block) j += a.second;
        return j;
    };
    const int x = rpu_index(rows_per_unit);
    return wl_sizes((size_t)c.ne_q, (size_t)(c.keys_q - joined(c.adj_q)), (size_t)c.nu_q[x] * heads) +
           wl_sizes((size_t)c.ne_kv, (size_t)(c.qrys_kv - joined(c.adj_kv)), (size_t)c.nu_kv[x] * heads);
}

size_t Planner::host_arena_bytes(int g, const PoolPlan &pl) const {
    const int64_t N = spec.N, R = max_task_rows;
    const size_t e = (size_t)spec.elem_bytes, dd = (size_t)spec.d;
    const size_t blk = (size_t)block * g * dd * e;
    const size_t blk_kv = (size_t)block * spec.kv_heads_of(g) * dd * e;  // fewer heads under GQA
    ArenaLayout a;
    a.take(256);                                        // error word
    a.take((size_t)N * g * dd * sizeof(float));         // accumulator O
    a.take((size_t)g * N * sizeof(float));              // accumulator lse
    a.take((size_t)pl.q_slots * blk);                   // Q block pool
    a.take((size_t)pl.kv_slots * blk_kv);               // K block pool
    a.take((size_t)pl.kv_slots * blk_kv);               // V block pool
    for (int s = 0; s < 2; ++s) {
        a.take((size_t)R * g * dd * e);                 // finished out rows
        a.take((size_t)g * R * sizeof(float));          // finished lse rows
    }
    for (int64_t t = 0; t < (int64_t)leaves.size(); ++t) a.take(leaf_wl_bytes(t, pl, unit_rows_for(spec.elem_bytes), g));
    return a.total;
}

// ---------------------------------------------------------------------------
// Resident schedule of the streamed forward (see planner.h, HostLaunch).
// ---------------------------------------------------------------------------
namespace {
constexpr int64_t kArrivalGroups = 16;  // copy-in marks per head group (fewer when there are fewer blocks)
constexpr int64_t kSms = 148;           // streaming multiprocessors of the B200
}

int64_t Planner::arrival_blocks() const {
    return std::max<int64_t>(1, (num_blocks + kArrivalGroups - 1) / kArrivalGroups);
}

std::vector<HostLaunch> Planner::host_launches(int rows_per_unit, int bn, int heads) const {
    const int64_t A = arrival_blocks();
    const int64_t G = (num_blocks + A - 1) / A;
    // Pairs needing one of the last quarter of the arrival groups are taken
    // query group by query group (the finishing phase).
    const int64_t cut = G - (G + 3) / 4;
    // Launch slots in order: for k < cut, [2k] = earlier query groups x keys
    // of group k, [2k + 1] = query group k x keys of groups <= k; then
    // [2 cut + j] = query group j's pairs of the finishing phase.  Per slot
    // and query block, the key blocks as inclusive intervals.
    const int64_t slots = 2 * cut + G;
    using Runs = std::vector<std::pair<int64_t, int64_t>>;
    std::vector<std::map<int64_t, Runs>> pairs(slots);
    for (const Entry &e : entries) {
        const int64_t gq = e.qb / A;
        for (const KeyRun &r : e.runs)
            for (int64_t b0 = r.b0; b0 <= r.b1;) {
                // the part of the run inside one arrival group
                const int64_t gk = b0 / A, b1 = std::min(r.b1, (gk + 1) * A - 1), w = std::max(gq, gk);
                const int64_t slot = w < cut ? 2 * w + (gq == w ? 1 : 0) : 2 * cut + gq;
                pairs[slot][e.qb].push_back({b0, b1});
                b0 = b1 + 1;
            }
    }
    // Finishing slots that need the same block go m query groups to a
    // launch, so that the two launches in flight (one per compute stream)
    // cover the SMs; slots that become ready at different arrivals (causal
    // plans) stay apart.
    const int64_t unit_per_group =
        (int64_t)heads * ((A * block + rows_per_unit - 1) / rows_per_unit);
    const int64_t m = std::max<int64_t>(1, (kSms / 2 + unit_per_group - 1) / unit_per_group);
    // Among slots ready at the same arrival, the longest chains of key
    // blocks go first, so that the phase ends on short ones.
    struct Fin {
        int64_t need, chain, sl;
    };
    std::vector<Fin> fin;
    for (int64_t sl = 2 * cut; sl < slots; ++sl) {
        if (pairs[sl].empty()) continue;
        Fin f{0, 0, sl};
        for (const auto &qk : pairs[sl]) {
            int64_t chain = 0;
            for (const auto &r : qk.second) {
                f.need = std::max(f.need, std::max(qk.first, r.second));
                chain += r.second - r.first + 1;
            }
            f.chain = std::max(f.chain, chain);
        }
        fin.push_back(f);
    }
    std::stable_sort(fin.begin(), fin.end(), [](const Fin &a, const Fin &b) {
        return a.need != b.need ? a.need < b.need : a.chain > b.chain;
    });
    std::vector<std::map<int64_t, Runs>> launch_pairs(pairs.begin(), pairs.begin() + 2 * cut);
    int64_t in_launch = 0, launch_need = -1;
    for (const Fin &f : fin) {
        const int64_t sl = f.sl, need = f.need;
        if (in_launch > 0 && in_launch < m && need == launch_need) {
            launch_pairs.back().insert(pairs[sl].begin(), pairs[sl].end());
            ++in_launch;
        } else {
            launch_pairs.push_back(std::move(pairs[sl]));
            in_launch = 1;
            launch_need = need;
        }
    }
    std::vector<HostLaunch> out;
    std::vector<int64_t> last(num_blocks, -1);  // latest launch that touched a query block
    std::vector<std::pair<int64_t, int32_t>> last_entry(num_blocks, {-1, -1});  // (launch, entry)
    for (auto &lp : launch_pairs) {
        if (lp.empty()) continue;
        HostLaunch L;
        L.stream = (int32_t)(out.size() & 1);
        for (auto &qk : lp) {
            const int64_t qb = qk.first;
            Runs &kr = qk.second;
            std::sort(kr.begin(), kr.end());
            const int64_t prev = last[qb];
            if (prev >= 0 && out[prev].stream != L.stream) L.after = std::max<int32_t>(L.after, (int32_t)prev);
            WlEntry w{};
            w.q_lo = (int32_t)(qb * block);
            w.q_hi = (int32_t)block_end(qb);
            w.q_goff = 0;
            w.slot = 0;
            w.out_lo = w.q_lo;
            w.flags = prev < 0 ? SEG_FIRST : 0;
            w.run_begin = (int32_t)L.wl.runs.size();
            L.need = std::max(L.need, qb);
            for (size_t i = 0; i < kr.size(); ++i) {
                L.need = std::max(L.need, kr[i].second);
                if (i > 0 && kr[i].first == kr[i - 1].second + 1) {
                    L.wl.runs.back().k_hi = (int32_t)block_end(kr[i].second);
                } else {
                    WlRun x{};
                    x.k_lo = (int32_t)(kr[i].first * block);
                    x.k_hi = (int32_t)block_end(kr[i].second);
                    L.wl.runs.push_back(x);
                }
            }
            w.run_count = (int32_t)L.wl.runs.size() - w.run_begin;
            last[qb] = (int64_t)out.size();
            last_entry[qb] = {(int64_t)out.size(), (int32_t)L.wl.entries.size()};
            L.wl.entries.push_back(w);
        }
        out.push_back(std::move(L));
    }
    // The last launch of each query block finishes it; units once the flags
    // are final.
    for (int64_t qb = 0; qb < num_blocks; ++qb) {
        if (last_entry[qb].first < 0) continue;
        HostLaunch &L = out[last_entry[qb].first];
        L.wl.entries[last_entry[qb].second].flags |= SEG_LAST;
        L.finish.push_back(qb);
    }
    for (HostLaunch &L : out) {
        std::vector<int64_t> group;
        for (const WlEntry &e : L.wl.entries) group.push_back(e.q_lo / block);
        add_units(&L.wl, heads, rows_per_unit, bn, spec.causal, group);
    }
    return out;
}

size_t Planner::resident_arena_bytes(int g, int sets, std::vector<HostLaunch> *launches) const {
    const int64_t N = spec.N, rows = num_blocks * block;
    const size_t e = (size_t)spec.elem_bytes, dd = (size_t)spec.d;
    const size_t gk = (size_t)spec.kv_heads_of(g);
    ArenaLayout a;
    a.take(256);                                        // error word
    for (int st = 0; st < sets; ++st) {                 // one buffer set per head group in flight
        a.take((size_t)N * g * dd * sizeof(float));     // accumulator O
        a.take((size_t)g * N * sizeof(float));          // accumulator lse
        a.take((size_t)rows * g * dd * e);              // Q pool, one slot per block
        a.take((size_t)rows * gk * dd * e);             // K pool
        a.take((size_t)rows * gk * dd * e);             // V pool
        a.take((size_t)N * g * dd * e);                 // finished out rows
        a.take((size_t)g * N * sizeof(float));          // finished lse rows
    }
    launches->clear();
    if (spec.budget && a.total > spec.budget) return a.total;  // does not fit: no need for the launches
    *launches = host_launches(unit_rows_for(spec.elem_bytes), key_tile_for(spec.elem_bytes), g);
    for (const HostLaunch &L : *launches) a.take(wl_bytes(L.wl));
    return a.total;
}

void Planner::size_plan() {
    sizing = Sizing{};
    host_sched.clear();
    sizing.device_arena = device_arena_bytes();
    // Smallest and largest useful pools (a task and its predecessor must fit).
    std::vector<std::vector<int64_t>> nq, nkv;
    task_needs(*this, &nq, &nkv);
    auto span = [](const std::vector<std::vector<int64_t>> &need, int64_t *mn, int64_t *full) {
        std::vector<int64_t> all;
        *mn = 0;
        for (size_t t = 0; t < need.size(); ++t) {
            std::vector<int64_t> u = need[t];
            if (t > 0) u.insert(u.end(), need[t - 1].begin(), need[t - 1].end());
            std::sort(u.begin(), u.end());
            u.erase(std::unique(u.begin(), u.end()), u.end());
            *mn = std::max<int64_t>(*mn, (int64_t)u.size());
            all.insert(all.end(), need[t].begin(), need[t].end());
        }
        std::sort(all.begin(), all.end());
        all.erase(std::unique(all.begin(), all.end()), all.end());
        *full = (int64_t)all.size();
    };
    span(nq, &min_q_slots, &full_q_slots);
    span(nkv, &min_kv_slots, &full_kv_slots);

    const int kvg = spec.kv_group();
    // The resident schedule (every block of a head group on the device:
    // each crosses the host link once per group, and the copies overlap the
    // launches pair by pair).  First with two buffer sets at the largest
    // head group of at most half the heads whose arena fits (the next
    // group's copies overlap this group's launches, and the first launches
    // wait for half the bytes), else with one set at the largest group.
    for (int pass = 0; pass < 2 && !spec.host_tasks && !sizing.resident; ++pass)
        for (int g = spec.H; g >= 1; --g) {
        if (spec.H % g || (g % kvg != 0 && kvg % g != 0)) continue;
        const int sets = pass == 0 ? 2 : 1;
        if (sets == 2 && spec.H / g < 2) continue;
        std::vector<HostLaunch> sched;
        const size_t rb = resident_arena_bytes(g, sets, &sched);
        PoolPlan pp;
        if ((spec.budget && rb > spec.budget) || !plan_pool(full_q_slots, full_kv_slots, &pp)) continue;
        const size_t blk = (size_t)block * g * spec.d * spec.elem_bytes;
        const size_t blk_kv = (size_t)block * spec.kv_heads_of(g) * spec.d * spec.elem_bytes;
        int64_t nb_rows = 0;
        for (int64_t b = 0; b < num_blocks; ++b) nb_rows += block_rows(b) > 0;
        host_sched = std::move(sched);
        sizing.head_group = g;
        sizing.host_arena = rb;
        sizing.q_slots = sizing.kv_slots = num_blocks;
        sizing.resident = true;
        sizing.sets = sets;
        sizing.h2d = (size_t)nb_rows * (blk + 2 * blk_kv) * (size_t)(spec.H / g);
        pool = std::move(pp);
        break;
        }
    for (int g = spec.H; g >= 1 && !sizing.resident; --g) {
        if (spec.H % g) continue;
        // A head group covers whole key/value groups, or lies inside one.
        if (g % kvg != 0 && kvg % g != 0) continue;
        const size_t blk = (size_t)block * g * spec.d * spec.elem_bytes;
        const size_t blk_kv = (size_t)block * spec.kv_heads_of(g) * spec.d * spec.elem_bytes;
        int64_t qs = full_q_slots, kvs = full_kv_slots;
        PoolPlan pp;
        if (!plan_pool(qs, kvs, &pp)) continue;
        size_t bytes = host_arena_bytes(g, pp);
        if (spec.budget) {
            // Shrink the pools (K/V first, they take two blocks per slot)
            // until the arena fits, never below what a task pair needs.
            while (bytes > spec.budget && (qs > min_q_slots || kvs > min_kv_slots)) {
                const size_t over = bytes - spec.budget;
                int64_t drop_kv =
                    std::min<int64_t>(kvs - min_kv_slots, (int64_t)((over + 2 * blk_kv - 1) / (2 * blk_kv)));
                int64_t drop_q = 0;
                if (drop_kv <= 0) drop_q = std::min<int64_t>(qs - min_q_slots, (int64_t)((over + blk - 1) / blk));
                if (drop_kv <= 0 && drop_q <= 0) break;
                kvs -= std::max<int64_t>(drop_kv, 0);
                qs -= std::max<int64_t>(drop_q, 0);
                if (!plan_pool(qs, kvs, &pp)) { bytes = SIZE_MAX; break; }
                bytes = host_arena_bytes(g, pp);
            }
            if (bytes > spec.budget) continue;
        }
        sizing.head_group = g;
        sizing.host_arena = bytes;
        sizing.q_slots = qs;
        sizing.kv_slots = kvs;
        const size_t groups = (size_t)(spec.H / g);
        sizing.h2d = ((size_t)pp.q_copies * blk + 2 * (size_t)pp.kv_copies * blk_kv) * groups;
        pool = std::move(pp);
        break;
    }
    sizing.d2h = (size_t)spec.N * spec.H * spec.d * spec.elem_bytes + (size_t)spec.H * spec.N * sizeof(float);
    // A call runs the B sequences one after another on the same plan.
    sizing.h2d *= (size_t)spec.B;
    sizing.d2h *= (size_t)spec.B;
}

// ---------------------------------------------------------------------------
// Streamed backward: block cache with running gradient sums (see planner.h).
// ---------------------------------------------------------------------------
namespace {

// Blocks a leaf task touches in the backward (as query or key), member order.
std::vector<std::vector<int64_t>> bwd_task_blocks(const Planner &pl) {
    const size_t T = pl.leaves.size();
    std::vector<std::vector<int64_t>> out(T);
    std::vector<char> q, kv;
    for (size_t t = 0; t < T; ++t) {
        pl.leaf_needs((int64_t)t, &q, &kv);
        for (size_t m = 0; m < q.size(); ++m)
            if (q[m] || kv[m]) out[t].push_back(pl.leaves[t].blocks[m]);
    }
    return out;
}

// Units of a key-stationary list: every 'rows' key rows of an entry, per
// head, with the query tiles the causal rule leaves; longest first.
void add_units_kv(WorkList *wl, int heads, int rows, int bn, int causal) {
    std::vector<WlUnit> u;
    for (int32_t ei = 0; ei < (int32_t)wl->entries.size(); ++ei) {
        const WlEntry &e = wl->entries[ei];
        for (int h = 0; h < heads; ++h)
            for (int64_t k0 = e.q_lo; k0 < e.q_hi; k0 += rows) {
                WlUnit x{ei, (int32_t)k0, h, unit_query_tiles(e, wl->runs.data(), (int32_t)k0, causal, bn)};
                if (x.ntiles > 0) u.push_back(x);
            }
    }
    std::stable_sort(u.begin(), u.end(), [](const WlUnit &a, const WlUnit &b) {
        const int ca = a.ntiles / 32, cb = b.ntiles / 32;
        if (ca != cb) return ca > cb;
        return a.head < b.head;
    });
    wl->units.swap(u);
}

// Appends rows [lo, lo + n) with global offset goff to the entry's runs,
// joining it to the previous run when the rows continue it.
void push_run(WorkList *wl, int32_t run_begin, int32_t lo, int32_t n, int32_t goff) {
    if ((int32_t)wl->runs.size() > run_begin && wl->runs.back().k_hi == lo && wl->runs.back().k_goff == goff) {
        wl->runs.back().k_hi = lo + n;
        return;
    }
    WlRun x{};
    x.k_lo = lo;
    x.k_hi = lo + n;
    x.k_goff = goff;
    wl->runs.push_back(x);
}

}  // namespace

bool Planner::plan_bwd_cache(int64_t C, BwdCachePlan *out) const {
    const std::vector<std::vector<int64_t>> &tb = bwd_blocks_;
    const int64_t T = (int64_t)tb.size();
    std::vector<std::vector<int64_t>> uses(num_blocks);
    for (int64_t t = 0; t < T; ++t)
        for (int64_t b : tb[t]) uses[b].push_back(t);
    auto next_use = [&](int64_t b, int64_t t) -> int64_t {
        auto it = std::upper_bound(uses[b].begin(), uses[b].end(), t);
        return it == uses[b].end() ? INT64_MAX : *it;
    };
    BwdCachePlan cp;
    cp.slots = C;
    cp.copies.assign(T, {});
    cp.member_slot.assign(T, {});
    cp.finals.assign(T, {});
    std::vector<int64_t> held(C, -1);        // block whose rows the slot holds
    std::vector<char> done(num_blocks, 0), on_host(num_blocks, 0);
    std::vector<int32_t> slot_of(num_blocks, -1);
    // Free slots: the lowest index first (a finished block's slot is free
    // from two tasks after its last one).  Eviction candidates: as in the
    // forward cache (simulate above), a lazy max-heap of (next use, -slot)
    // over the slots of unfinished blocks neither this task nor the
    // previous one touches.
    std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> free_slots;
    for (int64_t sl = 0; sl < C; ++sl) free_slots.push(sl);
    std::vector<std::vector<int32_t>> freed(T + 2), rejoin(T + 2);
    std::vector<int64_t> key(C, -1), guard(C, -1);
    std::priority_queue<std::pair<int64_t, int64_t>> heap;
    auto protect = [&](int32_t sl, int64_t b, int64_t t) {
        guard[sl] = t + 1;
        key[sl] = next_use(b, t);
        rejoin[t + 2].push_back(sl);
    };
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t sl : freed[t]) free_slots.push(sl);
        for (int32_t sl : rejoin[t])
            if (held[sl] >= 0 && !done[held[sl]] && guard[sl] == t - 1) heap.push({key[sl], -(int64_t)sl});
        for (int64_t b : tb[t])
            if (slot_of[b] >= 0) protect(slot_of[b], b, t);
        for (int64_t b : tb[t]) {
            if (slot_of[b] >= 0) continue;
            int32_t slot = -1;
            int64_t evict = -1;
            if (!free_slots.empty()) {
                slot = (int32_t)free_slots.top();
                free_slots.pop();
            } else {
                while (!heap.empty()) {
                    const std::pair<int64_t, int64_t> top = heap.top();
                    heap.pop();
                    const int32_t sl = (int32_t)(-top.second);
                    const int64_t ob = held[sl];
                    if (ob >= 0 && !done[ob] && key[sl] == top.first && guard[sl] < t) {
                        slot = sl;
                        break;
                    }
                }
                if (slot < 0) return false;
                evict = held[slot];
                slot_of[evict] = -1;
                on_host[evict] = 1;
                ++cp.writebacks;
            }
            cp.copies[t].push_back(BwdCopy{b, slot, evict, on_host[b] ? 1 : 0});
            ++cp.loads;
            held[slot] = b;
            slot_of[b] = slot;
            protect(slot, b, t);
        }
        const std::vector<int64_t> &blocks = leaves[t].blocks;
        cp.member_slot[t].assign(blocks.size(), -1);
        for (size_t m = 0; m < blocks.size(); ++m) cp.member_slot[t][m] = slot_of[blocks[m]];
        for (int64_t b : tb[t])
            if (uses[b].back() == t) {
                done[b] = 1;
                cp.finals[t].push_back({b, slot_of[b]});
                freed[t + 2].push_back(slot_of[b]);
                slot_of[b] = -1;
            }
    }
    *out = std::move(cp);
    return true;
}

WorkList Planner::leaf_bwd_q_worklist(int64_t t, const BwdCachePlan &c, int rows_per_unit, int bn,
                                      int heads) const {
    WorkList wl;
    for (int64_t i = entry_begin_of_leaf_[t]; i < entry_begin_of_leaf_[t + 1]; ++i) {
        const Entry &e = entries[i];
        const int64_t sq = c.member_slot[t][e.mq];
        WlEntry w{};
        w.q_lo = (int32_t)(sq * block);
        w.q_hi = (int32_t)(sq * block + block_rows(e.qb));
        w.q_goff = (int32_t)((e.qb - sq) * block);
        w.slot = 0;
        w.out_lo = w.q_lo;  // the block's dQ sums share its slot rows
        w.flags = 0;
        w.run_begin = (int32_t)wl.runs.size();
        for (const KeyRun &r : e.runs)
            for (int64_t kb = r.b0; kb <= r.b1; ++kb) {
                const int64_t sk = c.member_slot[t][r.m0 + (kb - r.b0)];
                push_run(&wl, w.run_begin, (int32_t)(sk * block), (int32_t)block_rows(kb),
                         (int32_t)((kb - sk) * block));
            }
        w.run_count = (int32_t)wl.runs.size() - w.run_begin;
        wl.entries.push_back(w);
    }
    add_units(&wl, heads, rows_per_unit, bn, spec.causal, std::vector<int64_t>(wl.entries.size(), t));
    return wl;
}

WorkList Planner::leaf_bwd_kv_worklist(int64_t t, const BwdCachePlan &c, int rows_per_unit, int bn,
                                       int heads) const {
    // key member -> query members whose entries' runs hold it
    const size_t n = leaves[t].blocks.size();
    std::vector<std::vector<int32_t>> qs_of(n);
    for (int64_t i = entry_begin_of_leaf_[t]; i < entry_begin_of_leaf_[t + 1]; ++i) {
        const Entry &e = entries[i];
        for (const KeyRun &r : e.runs)
            for (int64_t kb = r.b0; kb <= r.b1; ++kb) qs_of[r.m0 + (kb - r.b0)].push_back(e.mq);
    }
    WorkList wl;
    for (size_t mk = 0; mk < n; ++mk) {
        if (qs_of[mk].empty()) continue;
        std::vector<int32_t> &qm = qs_of[mk];
        std::sort(qm.begin(), qm.end());
        const int64_t kb = leaves[t].blocks[mk], sk = c.member_slot[t][mk];
        WlEntry w{};
        w.q_lo = (int32_t)(sk * block);
        w.q_hi = (int32_t)(sk * block + block_rows(kb));
        w.q_goff = (int32_t)((kb - sk) * block);
        w.slot = 0;
        w.out_lo = w.q_lo;  // the block's dK / dV sums share its slot rows
        w.flags = 0;
        w.run_begin = (int32_t)wl.runs.size();
        for (int32_t m : qm) {
            const int64_t qb = leaves[t].blocks[m], sq = c.member_slot[t][m];
            push_run(&wl, w.run_begin, (int32_t)(sq * block), (int32_t)block_rows(qb),
                     (int32_t)((qb - sq) * block));
        }
        w.run_count = (int32_t)wl.runs.size() - w.run_begin;
        wl.entries.push_back(w);
    }
    add_units_kv(&wl, heads, rows_per_unit, bn, spec.causal);
    // Grouped-query attention: units by query head modulo the group size, so
    // that each launch takes the query heads of one residue and no two of a
    // launch's CTAs add into the same key/value head's sums.
    const int kvg = spec.kv_group();
    if (kvg > 1)
        std::stable_sort(wl.units.begin(), wl.units.end(),
                         [kvg](const WlUnit &a, const WlUnit &b) { return a.head % kvg < b.head % kvg; });
    return wl;
}

size_t Planner::bwd_arena_bytes(int g, const BwdCachePlan &c) const {
    const size_t e = (size_t)spec.elem_bytes, dd = (size_t)spec.d, N = (size_t)spec.N;
    const size_t rows = (size_t)c.slots * block;
    const size_t gk = (size_t)(g / spec.kv_group());  // key/value heads of the group
    const int tile = spec.elem_bytes == 2 ? 128 : 64;
    ArenaLayout a;
    a.take(256);                                  // error word
    a.take((size_t)g * N * sizeof(float));        // lse of the head group
    a.take((size_t)g * N * sizeof(float));        // D = rowsum(dO * O)
    for (int s = 0; s < 4; ++s) a.take((size_t)block * g * dd * e);  // O / dO staging, two stages
    a.take(rows * g * dd * e);                    // Q pool
    a.take(rows * gk * dd * e);                   // K pool
    a.take(rows * gk * dd * e);                   // V pool
    a.take(rows * g * dd * e);                    // dO pool
    a.take(rows * g * dd * sizeof(float));        // dQ sums
    a.take(rows * gk * dd * sizeof(float));       // dK sums
    a.take(rows * gk * dd * sizeof(float));       // dV sums
    for (int64_t t = 0; t < (int64_t)leaves.size(); ++t) {
        // The two lists are laid out one after the other; each ArenaLayout
        // step is 256-aligned, so their sum is the same as two takes.
        a.take(leaf_bwd_wl_bytes(t, c, tile, g));
    }
    return a.total;
}

void Planner::size_bwd() {
    bwd_sizing = BwdSizing{};
    bwd_cache = BwdCachePlan{};
    // Head groups cover whole key/value groups, so that a key/value head's
    // sums collect all of its query heads' terms within one head group.
    if (spec.shard_count > 1) return;
    const int kvg = spec.kv_group();
    const std::vector<std::vector<int64_t>> tb = bwd_task_blocks(*this);
    bwd_min_slots = 0;
    std::vector<int64_t> all;
    for (size_t t = 0; t < tb.size(); ++t) {
        std::vector<int64_t> u = tb[t];
        if (t > 0) u.insert(u.end(), tb[t - 1].begin(), tb[t - 1].end());
        std::sort(u.begin(), u.end());
        u.erase(std::unique(u.begin(), u.end()), u.end());
        bwd_min_slots = std::max<int64_t>(bwd_min_slots, (int64_t)u.size());
        all.insert(all.end(), tb[t].begin(), tb[t].end());
    }
    std::sort(all.begin(), all.end());
    all.erase(std::unique(all.begin(), all.end()), all.end());
    bwd_full_slots = (int64_t)all.size();
    if (bwd_min_slots == 0) return;
    // For each head group g dividing H: the most slots that fit the budget;
    // keep the sizing that moves the fewest bytes over the host link (ties
    // to the larger group).
    double best_traffic = -1;
    for (int g = spec.H; g >= 1; --g) {
        if (spec.H % g || g % kvg) continue;
        if (!spec.budget && g < spec.H) break;  // unlimited: all heads at once, every block cached
        BwdCachePlan cp;
        int64_t C = bwd_full_slots;
        if (!plan_bwd_cache(C, &cp)) continue;
        size_t bytes = bwd_arena_bytes(g, cp);
        if (spec.budget && bytes > spec.budget) {
            // Largest C in [min, full) whose arena fits (bytes grow with C).
            int64_t lo = bwd_min_slots, hi = bwd_full_slots - 1, fit = -1;
            while (lo <= hi) {
                const int64_t mid = (lo + hi) / 2;
                BwdCachePlan m;
                if (plan_bwd_cache(mid, &m) && bwd_arena_bytes(g, m) <= spec.budget) {
                    fit = mid;
                    lo = mid + 1;
                } else {
                    hi = mid - 1;
                }
            }
            if (fit < 0) continue;
            C = fit;
            plan_bwd_cache(C, &cp);
            bytes = bwd_arena_bytes(g, cp);
        }
        const size_t gh = (size_t)g + (size_t)(g / kvg);  // heads of (Q, dO) and of (K, V): per pair
        const size_t blk = (size_t)block * spec.d * spec.elem_bytes;     // one head of one block
        const size_t acc = (size_t)block * spec.d * sizeof(float);
        const size_t groups = (size_t)(spec.H / g);
        const size_t N = (size_t)spec.N;
        const size_t sums = (size_t)g + 2 * (size_t)(g / kvg);             // heads of dQ, dK, dV
        const size_t h2d = groups * ((size_t)g * N * sizeof(float) + 2 * N * g * spec.d * spec.elem_bytes +
                                     (size_t)cp.loads * 2 * gh * blk + (size_t)cp.writebacks * sums * acc);
        const size_t d2h = groups * (N * sums * spec.d * spec.elem_bytes + (size_t)cp.writebacks * sums * acc);
        const double traffic = (double)h2d + (double)d2h;
        if (best_traffic < 0 || traffic < best_traffic) {
            best_traffic = traffic;
            bwd_sizing.head_group = g;
            bwd_sizing.arena = bytes;
            bwd_sizing.slots = C;
            bwd_sizing.h2d = h2d * (size_t)spec.B;
            bwd_sizing.d2h = d2h * (size_t)spec.B;
            bwd_sizing.spill_host = cp.writebacks ? N * sums * spec.d * sizeof(float) : 0;
            bwd_cache = std::move(cp);
        }
    }
}

ShardLayout Planner::shard_layout(int elem_bytes) const {
    ShardLayout L;
    L.G = std::max(1, spec.shard_count);
    L.me = spec.shard_rank;
    const int G = L.G;
    const int64_t H = spec.H, d = spec.d;
    L.owner.resize(num_blocks);
    for (int64_t b = 0; b < num_blocks; ++b) L.owner[b] = (int32_t)(b * G / num_blocks);
    L.row_lo.assign(G + 1, spec.N);
    for (int64_t b = num_blocks - 1; b >= 0; --b) L.row_lo[L.owner[b]] = std::min<int64_t>(b * block, spec.N);
    for (int k = G - 1; k >= 0; --k) L.row_lo[k] = std::min(L.row_lo[k], L.row_lo[k + 1]);
    for (int k = 0; k < G; ++k) L.rows_max = std::max(L.rows_max, L.row_lo[k + 1] - L.row_lo[k]);
    // touched[r * num_blocks + b]: rank r has an entry for query block b.
    std::vector<char> touched((size_t)G * num_blocks, 0);
    for (size_t i = 0; i < entries.size(); ++i) touched[(size_t)entry_rank[i] * num_blocks + entries[i].qb] = 1;
    // o rows, then lse padded to four floats: every piece starts 16-byte aligned.
    auto piece = [&](int64_t b) { return block_rows(b) * H * d + ((block_rows(b) * H + 3) & ~int64_t(3)); };
    L.send_counts.assign(G, 0);
    L.recv_counts.assign(G, 0);
    int64_t off = 0;
    for (int k = 0; k < G; ++k)
        for (int64_t b = 0; b < num_blocks; ++b)
            if (L.owner[b] == k && touched[(size_t)L.me * num_blocks + b] && block_rows(b) > 0) {
                L.send.push_back(ShardPiece{b, off});
                off += piece(b);
                L.send_counts[k] += piece(b);
            }
    L.own_first = num_blocks;
    for (int64_t b = 0; b < num_blocks; ++b)
        if (L.owner[b] == L.me) {
            L.own_first = std::min(L.own_first, b);
            ++L.own_count;
        }
    if (L.own_count == 0) L.own_first = 0;
    L.own_offsets.assign(L.own_count, {});
    off = 0;
    for (int r = 0; r < G; ++r)
        for (int64_t i = 0; i < L.own_count; ++i) {
            const int64_t b = L.own_first + i;
            if (touched[(size_t)r * num_blocks + b] && block_rows(b) > 0) {
                L.own_offsets[i].push_back(off);
                off += piece(b);
                L.recv_counts[r] += piece(b);
            }
        }
    auto up16 = [](size_t x) { return (x + 15) & ~size_t(15); };
    L.out_bytes = up16((size_t)L.rows_max * H * d * elem_bytes);
    L.chunk_bytes = L.out_bytes + up16((size_t)H * L.rows_max * sizeof(float));
    if (L.chunk_bytes == 0) L.chunk_bytes = 16;
    return L;
}

}  // namespace cqsa
