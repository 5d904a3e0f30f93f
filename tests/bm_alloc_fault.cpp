// Allocation-failure harness for the host block manager (include/pa_block_manager.h).
//
// Global operator new is replaced by one that throws std::bad_alloc at a chosen
// allocation.  A seeded script of manager calls (allocate, fork, append, free, swap
// out / in, under a sliding window or not) first runs without failures and records
// every call's status and outputs.  Then, for k = 0, 1, 2, ... until the script makes
// fewer than k allocations, the script runs again with the k-th allocation made inside
// a manager call failing.  The call that meets the failure must return
// PA_ERR_HOST_ALLOC (pa_bm_create: NULL) and leave everything the interface can observe
// unchanged; repeated without the failure it must give what it gave in the recorded
// run, and so must every later call.  Host only: no CUDA call, no GPU.
//
// Build: g++ -std=c++17 -I include tests/bm_alloc_fault.cpp
//            paged_kv_cache_441_b200/csrc/pa_block_manager.cpp
// Prints "ok <runs> <failures injected>" and exits 0, or prints the first mismatch
// and exits 1.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <random>
#include <string>
#include <vector>

#include "pa_block_manager.h"

namespace {
long g_countdown = -1;  // allocations until the failing one; -1 = none armed
bool g_armed = false;   // only allocations inside manager calls count
bool g_fired = false;
}  // namespace

void *operator new(std::size_t n) {
    if (g_armed && g_countdown >= 0) {
        if (g_countdown == 0) {
            g_countdown = -1;
            g_fired = true;
            throw std::bad_alloc();
        }
        --g_countdown;
    }
    void *p = std::malloc(n ? n : 1);
    if (!p) throw std::bad_alloc();
    return p;
}
void *operator new[](std::size_t n) { return operator new(n); }
void operator delete(void *p) noexcept { std::free(p); }
void operator delete[](void *p) noexcept { std::free(p); }
void operator delete(void *p, std::size_t) noexcept { std::free(p); }
void operator delete[](void *p, std::size_t) noexcept { std::free(p); }

namespace {

constexpr int kNb = 24, kBs = 4, kNcpu = 12, kOps = 160, kMaxIds = 64;

// Everything the interface shows about a manager.
struct Snapshot {
    std::vector<long long> v;
    bool operator==(const Snapshot &o) const { return v == o.v; }
};

Snapshot snap(const pa_block_manager *bm, int ids) {
    Snapshot s;
    s.v.push_back(pa_bm_num_free_blocks(bm));
    s.v.push_back(pa_bm_num_free_cpu_blocks(bm));
    s.v.push_back((long long)(pa_bm_usage_ratio(bm) * 1e9));
    for (int b = 0; b < kNb; ++b) s.v.push_back(pa_bm_block_refcount(bm, b));
    std::vector<int32_t> row(kNb + 1);
    for (int64_t id = 0; id < ids; ++id) {
        s.v.push_back(pa_bm_seq_len(bm, id));
        const int sw = pa_bm_is_swapped(bm, id);
        s.v.push_back(sw);
        if (sw == 0) {
            int32_t len = 0;
            s.v.push_back(pa_bm_block_tables(bm, &id, 1, row.data(), kNb + 1, &len));
            for (int32_t x : row) s.v.push_back(x);
            for (int pos = 0; pos < len; ++pos) s.v.push_back(pa_bm_slot(bm, id, pos));
        }
    }
    return s;
}

// One call's visible result: status and output arrays.
struct Result {
    std::vector<long long> v;
    bool operator==(const Result &o) const { return v == o.v; }
};

struct Op {
    int kind;  // 0 allocate, 1 fork, 2 append, 3 free, 4 swap out, 5 swap in
    std::vector<int64_t> ids;
    int n;
};

// The script: seeded, and independent of the results (calls that do not apply simply
// return an error, the same in every run).
std::vector<Op> script(unsigned seed) {
    std::mt19937 rng(seed);
    std::vector<Op> ops;
    int next = 0;
    for (int i = 0; i < kOps; ++i) {
        Op op;
        op.kind = (int)(rng() % 6);
        op.n = (int)(rng() % (3 * kBs + 2));
        const int span = next > 0 ? next : 1;
        if (op.kind == 0 || op.kind == 1) {
            if (next >= kMaxIds) op.kind = 2;
        }
        if (op.kind == 0) {
            op.ids = {next++};
        } else if (op.kind == 1) {
            op.ids = {(int64_t)(rng() % span), next++};
        } else if (op.kind == 2) {
            const int m = 1 + (int)(rng() % 4);
            for (int j = 0; j < m; ++j) op.ids.push_back((int64_t)(rng() % span));
        } else {
            const int m = 1 + (int)(rng() % 2);
            for (int j = 0; j < m; ++j) op.ids.push_back((int64_t)(rng() % span));
        }
        ops.push_back(op);
    }
    return ops;
}

int ids_after(const std::vector<Op> &ops, size_t upto) {
    int ids = 0;
    for (size_t i = 0; i < upto && i < ops.size(); ++i)
        if (ops[i].kind <= 1) ids = (int)ops[i].ids.back() + 1;
    return ids;
}

// The failure is armed (if `arm`) only around the manager call itself.
Result run_op(pa_block_manager *bm, const Op &op, bool arm) {
    Result r;
    r.v.reserve(2 + 4 * (2 * kNb + 2));
    const int n = (int)op.ids.size();
    std::vector<int64_t> a(2 * kNb + 2, -7), b(2 * kNb + 2, -7);
    int np = -1;
    pa_status st;
    g_armed = arm;
    switch (op.kind) {
        case 0: st = pa_bm_allocate(bm, op.ids[0], op.n); break;
        case 1: st = pa_bm_fork(bm, op.ids[0], op.ids[1]); break;
        case 2: st = pa_bm_append_slots(bm, op.ids.data(), n, a.data(), b.data(), kNb, &np); break;
        case 3: st = pa_bm_free(bm, op.ids[0]); break;
        case 4: st = pa_bm_swap_out(bm, op.ids.data(), n, a.data(), kNb, &np); break;
        default: st = pa_bm_swap_in(bm, op.ids.data(), n, a.data(), kNb, &np); break;
    }
    g_armed = false;
    r.v.push_back(st);
    r.v.push_back(np);
    r.v.insert(r.v.end(), a.begin(), a.end());
    r.v.insert(r.v.end(), b.begin(), b.end());
    return r;
}

// A pool, its host pool and window; NULL when a call failed (only by an injected
// failure, which the caller checks).
pa_block_manager *make(int window, bool arm) {
    g_armed = arm;
    pa_block_manager *bm = pa_bm_create(kNb, kBs);
    pa_status st = bm ? pa_bm_set_cpu_pool(bm, kNcpu) : PA_OK;
    if (bm && st == PA_OK) st = pa_bm_set_sliding_window(bm, window);
    g_armed = false;
    if (bm && st != PA_OK) {
        pa_bm_destroy(bm);
        return nullptr;
    }
    return bm;
}

int fail(const char *what, int window, long k, size_t i) {
    std::printf("FAIL %s (window %d, failing allocation %ld, call %zu)\n", what, window, k, i);
    return 1;
}

}  // namespace

int main() {
    long runs = 0, injected = 0;
    for (int window : {0, 6}) {
        const std::vector<Op> ops = script(1234u + (unsigned)window);
        // the recorded run
        std::vector<Result> want;
        pa_block_manager *ref = make(window, false);
        if (!ref) return fail("create without failures", window, -1, 0);
        for (const Op &op : ops) want.push_back(run_op(ref, op, false));
        const Snapshot want_end = snap(ref, ids_after(ops, ops.size()));
        pa_bm_destroy(ref);
        int ok_calls = 0;
        for (const Result &r : want) ok_calls += r.v[0] == PA_OK;
        if (ok_calls < kOps / 4) return fail("script too dull (few calls succeed)", window, -1, 0);

        for (long k = 0;; ++k) {
            ++runs;
            g_fired = false;
            g_countdown = k;
            // pool creation and set-up count too
            pa_block_manager *bm = make(window, true);
            if (!bm) {
                if (!g_fired) return fail("create returned NULL without a failure", window, k, 0);
                ++injected;
                continue;  // the failure hit creation; it returned NULL as documented
            }
            for (size_t i = 0; i < ops.size(); ++i) {
                const int ids = ids_after(ops, i + 1);
                const bool pending = g_countdown >= 0;
                Snapshot before;
                if (pending) before = snap(bm, ids);
                Result got = run_op(bm, ops[i], true);
                if (g_fired && pending && g_countdown < 0) {
                    // this call met the failure
                    g_fired = false;
                    ++injected;
                    if (got.v[0] != PA_ERR_HOST_ALLOC)
                        return fail("a failed allocation did not return PA_ERR_HOST_ALLOC",
                                    window, k, i);
                    if (!(snap(bm, ids) == before))
                        return fail("a call that failed changed the manager", window, k, i);
                    got = run_op(bm, ops[i], false);  // again, without a failure
                }
                if (!(got == want[i])) return fail("result differs from the recorded run", window, k, i);
            }
            const Snapshot end = snap(bm, ids_after(ops, ops.size()));
            pa_bm_destroy(bm);
            if (!(end == want_end)) return fail("final state differs", window, k, ops.size());
            if (g_countdown >= 0) break;  // fewer than k allocations: every one was tried
        }
    }
    std::printf("ok %ld %ld\n", runs, injected);
    return 0;
}
