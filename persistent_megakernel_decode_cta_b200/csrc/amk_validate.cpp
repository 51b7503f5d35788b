// amk_validate.cpp -- static validator for per-SM task schedules.
//
// x-techcon "AutoMegaKernel ... persistent cooperative kernel", section 1
// (statically verified schedule IR) and the gist.science technical summary,
// "De Safety Gate": before any launch a frozen validator checks the typed
// task DAG -- wait thresholds between 1 and the producer count, an acyclic
// producer/consumer graph, per-SM queues that are linear extensions of the
// DAG, multi-producer counters waited only at full count, and every reader's
// writer a topological predecessor -- so an unsafe schedule is REJECTED
// instead of hanging the GPU ("RightNow-AI/AutoMegaKernel" README,
// "Deadlock-free by construction").
//
// Readings taken here (the pages list the checks, not their algorithms):
//  * "linear extension" is checked on the union of counter edges and queue
//    edges: some global topological order must contain every queue as a
//    subsequence, which is exactly the condition under which the per-SM
//    loops cannot deadlock.
//  * "happens before" is reachability in that union graph.
//  * A flagged read (the task polls the words themselves, each carrying the
//    epoch's tag once its one writer stored it or its accumulators finished)
//    is a wait on every task with a WRITE or ACCUM overlapping the range: it
//    adds those edges to the graph (rule V10 makes sure there is exactly one
//    value to wait for).
//  * The pages' reader/writer rule is extended with the other conflicts a
//    single-assignment step can have (write/write, accumulate, the previous
//    step's value, resets for the next step) and with a coverage rule for
//    double-buffered accumulators (rules V6, V9 in amk.h).
#include <algorithm>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "amk.h"
#include "amk_internal.h"

namespace {

struct Fail {
    amk_validation_report *rep;
    int operator()(int rule, int a, int b, int ctr, int buf, const char *fmt, ...)
    {
        if (rep) {
            rep->rule = rule;
            rep->task_a = a;
            rep->task_b = b;
            rep->counter = ctr;
            rep->buffer = buf;
            va_list ap;
            va_start(ap, fmt);
            vsnprintf(rep->message, sizeof rep->message, fmt, ap);
            va_end(ap);
        }
        return AMK_ERR_VALIDATION;
    }
};

bool in(int64_t v, int64_t lo, int64_t hi) { return v >= lo && v < hi; }

// Kahn's algorithm; returns true if acyclic and fills topo order.
bool topo_sort(int n, const std::vector<std::vector<int>> &succ, std::vector<int> &order,
               int *stuck)
{
    std::vector<int> indeg(n, 0);
    for (int u = 0; u < n; ++u)
        for (int v : succ[u])
            ++indeg[v];
    order.clear();
    order.reserve(n);
    for (int u = 0; u < n; ++u)
        if (indeg[u] == 0)
            order.push_back(u);
    for (size_t i = 0; i < order.size(); ++i)
        for (int v : succ[order[i]])
            if (--indeg[v] == 0)
                order.push_back(v);
    if ((int)order.size() == n)
        return true;
    for (int u = 0; u < n; ++u)
        if (indeg[u] > 0) {
            *stuck = u;
            break;
        }
    return false;
}

struct Acc {
    int task, kind;
    int64_t b, e;
};

}  // namespace

extern "C" int amk_validate_graph(const amk_graph *g, amk_validation_report *rep)
{
    if (!g)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_validate_graph: graph is NULL");
    if (rep) {
        memset(rep, 0, sizeof *rep);
        rep->task_a = rep->task_b = rep->counter = rep->buffer = -1;
    }
    Fail fail{rep};
    const int T = g->n_tasks, C = g->n_counters, B = g->n_buffers, S = g->n_sms;
    if (T < 0 || C < 0 || B < 0 || S < 0 || g->n_waits < 0 || g->n_signals < 0 ||
        g->n_accesses < 0)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_validate_graph: negative count");

    // ---- V7: referential integrity -------------------------------------
    if ((T > 0 && !g->tasks) || (g->n_waits > 0 && !g->waits) ||
        (g->n_signals > 0 && !g->signals) || (g->n_accesses > 0 && !g->accesses) ||
        (B > 0 && !g->buffers) || (T > 0 && (!g->queue_tasks || S < 1)) ||
        (S > 0 && !g->queue_offsets))
        return fail(AMK_RULE_V7, -1, -1, -1, -1, "missing array");
    for (int b = 0; b < B; ++b) {
        const amk_graph_buffer &bf = g->buffers[b];
        if (bf.size < 0 || (bf.pair != -1 && (!in(bf.pair, 0, B) || bf.pair == b)))
            return fail(AMK_RULE_V7, -1, -1, -1, b, "buffer %d: bad size or pair", b);
    }
    if (S > 0) {
        if (g->queue_offsets[0] != 0 || g->queue_offsets[S] != T)
            return fail(AMK_RULE_V7, -1, -1, -1, -1, "queue offsets do not span the tasks");
        for (int s = 0; s < S; ++s)
            if (g->queue_offsets[s + 1] < g->queue_offsets[s])
                return fail(AMK_RULE_V7, -1, -1, -1, -1, "queue offsets decrease at sm %d", s);
    }
    {
        std::vector<char> seen(T, 0);
        for (int s = 0; s < S; ++s)
            for (int i = g->queue_offsets[s]; i < g->queue_offsets[s + 1]; ++i) {
                int t = g->queue_tasks[i];
                if (!in(t, 0, T))
                    return fail(AMK_RULE_V7, t, -1, -1, -1, "queue of sm %d names task %d", s, t);
                if (seen[t])
                    return fail(AMK_RULE_V7, t, -1, -1, -1, "task %d queued twice", t);
                seen[t] = 1;
                if (g->tasks[t].sm != s)
                    return fail(AMK_RULE_V7, t, -1, -1, -1, "task %d is in the queue of sm %d "
                                "but names sm %d", t, s, g->tasks[t].sm);
            }
    }
    for (int t = 0; t < T; ++t) {
        const amk_graph_task &k = g->tasks[t];
        if (k.wait_count < 0 || k.signal_count < 0 || k.access_count < 0 ||
            k.wait_begin < 0 || k.wait_begin + (int64_t)k.wait_count > g->n_waits ||
            k.signal_begin < 0 || k.signal_begin + (int64_t)k.signal_count > g->n_signals ||
            k.access_begin < 0 || k.access_begin + (int64_t)k.access_count > g->n_accesses)
            return fail(AMK_RULE_V7, t, -1, -1, -1, "task %d: list out of range", t);
        for (int i = 0; i < k.wait_count; ++i)
            if (!in(g->waits[k.wait_begin + i].counter, 0, C))
                return fail(AMK_RULE_V7, t, -1, g->waits[k.wait_begin + i].counter, -1,
                            "task %d waits on a missing counter", t);
        for (int i = 0; i < k.signal_count; ++i)
            if (!in(g->signals[k.signal_begin + i], 0, C))
                return fail(AMK_RULE_V7, t, -1, g->signals[k.signal_begin + i], -1,
                            "task %d signals a missing counter", t);
        for (int i = 0; i < k.access_count; ++i) {
            const amk_graph_access &a = g->accesses[k.access_begin + i];
            if (!in(a.buffer, 0, B))
                return fail(AMK_RULE_V7, t, -1, -1, a.buffer, "task %d names a missing buffer", t);
            if (a.kind < AMK_ACC_READ || a.kind > AMK_ACC_READ_FLAGGED)
                return fail(AMK_RULE_V7, t, -1, -1, a.buffer, "task %d: bad access kind", t);
            if (a.begin < 0 || a.end <= a.begin || a.end > g->buffers[a.buffer].size)
                return fail(AMK_RULE_V7, t, -1, -1, a.buffer,
                            "task %d: range [%lld,%lld) outside buffer %d", t,
                            (long long)a.begin, (long long)a.end, a.buffer);
        }
    }

    // ---- V2 / V3: thresholds ---------------------------------------------
    std::vector<int> producers(C, 0);
    for (int t = 0; t < T; ++t)
        for (int i = 0; i < g->tasks[t].signal_count; ++i)
            ++producers[g->signals[g->tasks[t].signal_begin + i]];
    for (int t = 0; t < T; ++t) {
        const amk_graph_task &k = g->tasks[t];
        for (int i = 0; i < k.wait_count; ++i) {
            const amk_graph_wait &w = g->waits[k.wait_begin + i];
            if (w.threshold < 1 || w.threshold > producers[w.counter])
                return fail(AMK_RULE_V2, t, -1, w.counter, -1,
                            "task %d waits on counter %d for %d of %d producers", t, w.counter,
                            w.threshold, producers[w.counter]);
        }
    }
    for (int t = 0; t < T; ++t) {
        const amk_graph_task &k = g->tasks[t];
        for (int i = 0; i < k.wait_count; ++i) {
            const amk_graph_wait &w = g->waits[k.wait_begin + i];
            if (producers[w.counter] > 1 && w.threshold != producers[w.counter])
                return fail(AMK_RULE_V3, t, -1, w.counter, -1,
                            "task %d partially waits (%d of %d) on shared counter %d", t,
                            w.threshold, producers[w.counter], w.counter);
        }
    }

    // accesses per buffer (sorted by start, then task)
    std::vector<std::vector<Acc>> per_buf(B);
    for (int t = 0; t < T; ++t) {
        const amk_graph_task &k = g->tasks[t];
        for (int i = 0; i < k.access_count; ++i) {
            const amk_graph_access &a = g->accesses[k.access_begin + i];
            per_buf[a.buffer].push_back({t, a.kind, a.begin, a.end});
        }
    }
    for (auto &v : per_buf)
        std::sort(v.begin(), v.end(), [](const Acc &x, const Acc &y) {
            return x.b != y.b ? x.b < y.b : x.task < y.task;
        });
    auto is_w = [](int k) { return k == AMK_ACC_WRITE || k == AMK_ACC_ACCUM; };

    // ---- V10: flagged reads find exactly one value per element ---------------
    for (int b = 0; b < B; ++b) {
        const auto &v = per_buf[b];
        bool any = false;
        for (const Acc &a : v)
            any |= a.kind == AMK_ACC_READ_FLAGGED;
        if (!any)
            continue;
        const int64_t n = g->buffers[b].size;
        std::vector<int64_t> dw(n + 1, 0), da(n + 1, 0);  // difference arrays
        for (const Acc &a : v) {
            if (a.kind == AMK_ACC_WRITE)
                ++dw[a.b], --dw[a.e];
            else if (a.kind == AMK_ACC_ACCUM)
                ++da[a.b], --da[a.e];
        }
        std::vector<int64_t> bad(n + 1, 0);  // prefix count of elements without one value
        int64_t cw = 0, ca = 0;
        for (int64_t x = 0; x < n; ++x) {
            cw += dw[x];
            ca += da[x];
            const bool ok = (cw == 1 && ca == 0) || (cw == 0 && ca >= 1);
            bad[x + 1] = bad[x] + (ok ? 0 : 1);
        }
        for (const Acc &a : v)
            if (a.kind == AMK_ACC_READ_FLAGGED && bad[a.e] != bad[a.b])
                return fail(AMK_RULE_V10, a.task, -1, -1, b,
                            "task %d reads flagged elements of buffer %d in [%lld,%lld) that "
                            "are not written exactly once (or only accumulated)", a.task, b,
                            (long long)a.b, (long long)a.e);
    }

    // ---- V1 / V4: acyclicity -------------------------------------------------
    // nodes: tasks [0, T), counters [T, T+C), then one join node per set of
    // more than kDirect writers that a flagged read waits for (edges writer ->
    // join -> reader, like a counter's); smaller sets get direct edges
    constexpr size_t kDirect = 8;
    std::vector<std::vector<int>> succ(T + C);
    for (int t = 0; t < T; ++t) {
        const amk_graph_task &k = g->tasks[t];
        for (int i = 0; i < k.signal_count; ++i)
            succ[t].push_back(T + g->signals[k.signal_begin + i]);
        for (int i = 0; i < k.wait_count; ++i)
            succ[T + g->waits[k.wait_begin + i].counter].push_back(t);
    }
    {
        std::vector<std::pair<std::vector<int>, int>> joins;  // writer set -> node
        for (int b = 0; b < B; ++b) {
            const auto &v = per_buf[b];
            for (const Acc &r : v) {
                if (r.kind != AMK_ACC_READ_FLAGGED)
                    continue;
                std::vector<int> ws;
                for (const Acc &w : v)
                    if (is_w(w.kind) && w.b < r.e && r.b < w.e)
                        ws.push_back(w.task);
                std::sort(ws.begin(), ws.end());
                ws.erase(std::unique(ws.begin(), ws.end()), ws.end());
                if (ws.size() <= kDirect) {
                    for (int w : ws)
                        succ[w].push_back(r.task);
                    continue;
                }
                int node = -1;
                for (const auto &j : joins)
                    if (j.first == ws) {
                        node = j.second;
                        break;
                    }
                if (node < 0) {
                    node = (int)succ.size();
                    succ.emplace_back();
                    for (int w : ws)
                        succ[w].push_back(node);
                    joins.push_back({ws, node});
                }
                succ[node].push_back(r.task);
            }
        }
    }
    const int N = (int)succ.size();
    std::vector<int> order;
    int stuck = -1;
    if (!topo_sort(N, succ, order, &stuck))
        return fail(AMK_RULE_V1, stuck < T ? stuck : -1, -1,
                    stuck >= T && stuck < T + C ? stuck - T : -1, -1,
                    "producer/consumer graph has a cycle (through %s %d)",
                    stuck < T ? "task" : stuck < T + C ? "counter" : "flagged join",
                    stuck < T ? stuck : stuck < T + C ? stuck - T : stuck - T - C);
    for (int s = 0; s < S; ++s)
        for (int i = g->queue_offsets[s]; i + 1 < g->queue_offsets[s + 1]; ++i)
            succ[g->queue_tasks[i]].push_back(g->queue_tasks[i + 1]);
    if (!topo_sort(N, succ, order, &stuck))
        return fail(AMK_RULE_V4, stuck < T ? stuck : -1, -1, -1, -1,
                    "per-SM queue order contradicts the dependency graph (near %s %d)",
                    stuck < T ? "task" : stuck < T + C ? "counter" : "flagged join",
                    stuck < T ? stuck : stuck < T + C ? stuck - T : stuck - T - C);

    // ---- happens-before closure over tasks (bitsets in topological order) ---
    const size_t W = ((size_t)T + 63) / 64;
    std::vector<uint64_t> reach((size_t)N * W, 0);
    for (int u : order) {
        uint64_t *ru = &reach[(size_t)u * W];
        for (int v : succ[u]) {
            uint64_t *rv = &reach[(size_t)v * W];
            for (size_t w = 0; w < W; ++w)
                rv[w] |= ru[w];
            if (u < T)
                rv[u >> 6] |= 1ull << (u & 63);
        }
    }
    auto hb = [&](int a, int b) {  // a happens before b
        return (reach[(size_t)b * W + (a >> 6)] >> (a & 63)) & 1;
    };

    // ---- V5 / V6: conflicting accesses ---------------------------------------
    // (a READ_FLAGGED follows its writers by its own edges; it is checked as a
    // READ below, which it always passes, and against RESETs as any access)
    for (int pass = 5; pass <= 6; ++pass) {
        for (int b = 0; b < B; ++b) {
            const auto &v = per_buf[b];
            for (size_t i = 0; i < v.size(); ++i)
                for (size_t j = i + 1; j < v.size() && v[j].b < v[i].e; ++j) {
                    const Acc *x = &v[i], *y = &v[j];
                    if (x->task == y->task)
                        continue;
                    if (pass == 5) {
                        // every READ after every overlapping WRITE/ACCUM
                        for (int r = 0; r < 2; ++r, std::swap(x, y))
                            if ((x->kind == AMK_ACC_READ || x->kind == AMK_ACC_READ_FLAGGED) &&
                                is_w(y->kind) && !hb(y->task, x->task))
                                return fail(AMK_RULE_V5, y->task, x->task, -1, b,
                                            "task %d reads buffer %d before writer %d is "
                                            "ordered before it", x->task, b, y->task);
                        continue;
                    }
                    int kx = x->kind, ky = y->kind;
                    bool ordered = hb(x->task, y->task) || hb(y->task, x->task);
                    if (((kx == AMK_ACC_WRITE && is_w(ky)) || (ky == AMK_ACC_WRITE && is_w(kx)) ||
                         (kx == AMK_ACC_RESET && ky == AMK_ACC_RESET)) && !ordered)
                        return fail(AMK_RULE_V6, x->task, y->task, -1, b,
                                    "unordered writes to buffer %d by tasks %d and %d", b,
                                    x->task, y->task);
                    for (int r = 0; r < 2; ++r, std::swap(x, y)) {
                        int k1 = x->kind, k2 = y->kind;
                        if (k1 == AMK_ACC_READ_PREV &&
                            (is_w(k2) || k2 == AMK_ACC_RESET) && !hb(x->task, y->task))
                            return fail(AMK_RULE_V6, x->task, y->task, -1, b,
                                        "task %d reads the previous step's buffer %d but is "
                                        "not ordered before task %d's write", x->task, b,
                                        y->task);
                        if (k1 == AMK_ACC_RESET && k2 != AMK_ACC_RESET &&
                            !hb(y->task, x->task))
                            return fail(AMK_RULE_V6, y->task, x->task, -1, b,
                                        "task %d resets buffer %d without following task "
                                        "%d's access", x->task, b, y->task);
                    }
                }
        }
    }

    // ---- V8: outputs are produced -------------------------------------------
    for (int b = 0; b < B; ++b) {
        if (!(g->buffers[b].flags & AMK_BUF_OUTPUT))
            continue;
        bool written = false;
        for (const Acc &a : per_buf[b])
            written |= is_w(a.kind);
        if (!written)
            return fail(AMK_RULE_V8, -1, -1, -1, b, "output buffer %d is never written", b);
    }

    // ---- V9: next-step accumulators are reset ---------------------------------
    for (int b = 0; b < B; ++b) {
        int p = g->buffers[b].pair;
        if (p < 0)
            continue;
        std::vector<std::pair<int64_t, int64_t>> cover;
        for (const Acc &a : per_buf[p])
            if (a.kind == AMK_ACC_RESET)
                cover.push_back({a.b, a.e});
        std::sort(cover.begin(), cover.end());
        std::vector<std::pair<int64_t, int64_t>> merged;
        for (auto &iv : cover) {
            if (!merged.empty() && iv.first <= merged.back().second)
                merged.back().second = std::max(merged.back().second, iv.second);
            else
                merged.push_back(iv);
        }
        for (const Acc &a : per_buf[b]) {
            if (a.kind != AMK_ACC_ACCUM)
                continue;
            bool ok = false;
            for (auto &iv : merged)
                ok |= iv.first <= a.b && a.e <= iv.second;
            if (!ok)
                return fail(AMK_RULE_V9, a.task, -1, -1, b,
                            "task %d accumulates buffer %d range [%lld,%lld) that buffer %d's "
                            "resets do not cover", a.task, b, (long long)a.b, (long long)a.e, p);
        }
    }
    return AMK_OK;
}
