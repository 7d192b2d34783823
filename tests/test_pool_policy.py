"""The resident pool's slot policy (host logic, no GPU): a compiled driver runs the
library's SlotCache through batches and checks reuse, least-recently-used eviction,
that a batch never evicts its own keys, rejection of oversize batches, and drop.
Also the pool manager's host-side argument checks (no CUDA call is reached)."""
import ctypes
import os
import subprocess

import pytest

import adapter_gemv_sgmv_b200 as L
from adapter_gemv_sgmv_b200 import build as B

DRIVER = r'''
#include "slot_cache.h"
#include <cstdio>
#include <vector>
using lora::SlotCache;
static int fails = 0;
#define CHECK(c) do { if (!(c)) { std::printf("FAIL line %d: %s\n", __LINE__, #c); ++fails; } } while (0)
int main() {
    SlotCache c(3);
    std::vector<std::pair<int, int64_t>> L;
    int s[8];
    // first batch: three distinct keys fill the three slots in order of appearance
    int64_t b1[] = {10, 11, 10, 12};
    CHECK(c.assign(b1, 4, s, &L));
    CHECK(s[0] == 0 && s[1] == 1 && s[2] == 0 && s[3] == 2 && L.size() == 3);
    // a resident key keeps its slot; nothing loads
    int64_t b2[] = {11};
    CHECK(c.assign(b2, 1, s, &L) && s[0] == 1 && L.empty());
    // a new key replaces the least recently used slot (10 and 12 last used in batch 1; 10 first)
    int64_t b3[] = {13};
    CHECK(c.assign(b3, 1, s, &L) && s[0] == 0 && L.size() == 1 && L[0].second == 13);
    CHECK(c.find(10) == -1 && c.find(11) == 1 && c.find(12) == 2 && c.find(13) == 0);
    // a batch never evicts its own keys: {12, 14} must take slot 1 (key 11), not slot 2
    int64_t b4[] = {12, 14};
    CHECK(c.assign(b4, 2, s, &L) && s[0] == 2 && s[1] == 1 && L.size() == 1);
    // more distinct keys than slots: rejected, nothing changes
    int64_t b5[] = {1, 2, 3, 4};
    CHECK(!c.assign(b5, 4, s, &L));
    CHECK(c.find(12) == 2 && c.find(14) == 1 && c.find(13) == 0);
    // drop frees the slot; the next new key takes it
    c.drop(14);
    int64_t b6[] = {15};
    CHECK(c.assign(b6, 1, s, &L) && s[0] == 1);
    // an empty batch changes nothing
    CHECK(c.assign(b6, 0, s, &L) && L.empty());
    // a copy that fails part-way through a batch: the failing key and every later
    // key of the batch are rolled back (not resident), the earlier ones stay
    {
        SlotCache r(4);
        int64_t bb[] = {20, 21, 22, 23};
        CHECK(r.assign(bb, 4, s, &L) && L.size() == 4);
        r.rollback(L, 1);                   // the copy of loads[1] (key 21) failed
        CHECK(r.find(20) == 0 && r.find(21) == -1 && r.find(22) == -1 && r.find(23) == -1);
        // the next batch needing them loads them again, into the freed slots
        int64_t again[] = {21, 23};
        CHECK(r.assign(again, 2, s, &L) && L.size() == 2 && s[0] != 0 && s[1] != 0 && s[0] != s[1]);
        CHECK(r.find(20) == 0);
    }
    // co-occurrence: partners ranked by the requests they shared, ties to the smaller key
    {
        lora::CoOccurrence co;
        int64_t q1[] = {1, 2, 3}, q2[] = {1, 3}, q3[] = {1, 4, 4}, q4[] = {5};
        co.observe(q1, 3);
        co.observe(q2, 2);
        co.observe(q3, 3);                  // a duplicate key counts once
        co.observe(q4, 1);
        std::vector<int64_t> t;
        co.top(1, 2, &t);
        CHECK(t.size() == 2 && t[0] == 3 && t[1] == 2);     // 3 (twice), then 2 and 4 tie: 2
        co.top(1, 5, &t);
        CHECK(t.size() == 3 && t[2] == 4);
        CHECK(co.pairs(4, 1) == 1 && co.pairs(4, 4) == 0 && co.pairs(5, 1) == 0);
        co.top(5, 3, &t);
        CHECK(t.empty());
        co.top(9, 3, &t);
        CHECK(t.empty());
    }
    // preloading after a batch: free slots first, then least recently used ones, never a
    // key of this batch; stops when only the batch's slots are left
    {
        SlotCache p(4);
        int64_t b1[] = {1, 2};
        CHECK(p.assign(b1, 2, s, &L));
        int64_t pre1[] = {7, 8, 9};
        p.preload(pre1, 3, &L);              // two free slots: 7 and 8 come in, 9 does not fit
        CHECK(L.size() == 2 && p.find(7) == 2 && p.find(8) == 3 && p.find(9) == -1);
        CHECK(p.find(1) == 0 && p.find(2) == 1);
        int64_t b2[] = {7};                  // resident thanks to the preload: no load
        CHECK(p.assign(b2, 1, s, &L) && L.empty() && s[0] == 2);
        int64_t pre2[] = {9, 7};             // 9 evicts the least recently used key (1), 7 stays
        p.preload(pre2, 2, &L);
        CHECK(L.size() == 1 && L[0].second == 9 && p.find(9) == 0 && p.find(1) == -1 && p.find(7) == 2);
    }
    std::printf("fails %d\n", fails);
    return fails != 0;
}
'''

COVERAGE_DRIVER = r'''
#include "slot_cache.h"
#include <cstdio>
#include <fstream>
#include <sstream>
#include <string>
#include <vector>
// Reads one request's adapter list per line; prints, for k = 1..3, the coverage of
// top-k co-occurrence prediction (the share of a multi-adapter request's other
// adapters among the top k partners of its first one, counts from earlier requests
// only) and the hit rate of the other adapters in a 16-slot pool that acquires each
// request's first adapter with top-k preloading, then the rest.
int main(int argc, char **argv) {
    std::ifstream in(argv[1]);
    std::vector<std::vector<int64_t>> reqs;
    for (std::string line; std::getline(in, line);) {
        std::istringstream ss(line);
        std::vector<int64_t> r;
        for (int64_t v; ss >> v;) r.push_back(v);
        if (!r.empty()) reqs.push_back(r);
    }
    for (int k = 0; k <= 3; ++k) {
        lora::CoOccurrence co;
        lora::SlotCache cache(16);
        std::vector<std::pair<int, int64_t>> loads;
        std::vector<int64_t> top;
        double cov = 0, n_multi = 0, hits = 0, others = 0;
        int slots[8];
        for (const auto &r : reqs) {
            co.top(r[0], k, &top);
            if (r.size() > 1) {
                int in_top = 0;
                for (size_t i = 1; i < r.size(); ++i)
                    for (int64_t t : top) in_top += (t == r[i]);
                cov += (double)in_top / (double)(r.size() - 1);
                n_multi += 1;
            }
            cache.assign(&r[0], 1, slots, &loads);
            std::vector<int64_t> want;
            for (int64_t t : top) if (t != r[0]) want.push_back(t);
            cache.preload(want.data(), (int)want.size(), &loads);
            for (size_t i = 1; i < r.size(); ++i) { hits += cache.find(r[i]) >= 0; others += 1; }
            cache.assign(r.data(), (int)r.size(), slots, &loads);
            co.observe(r.data(), (int)r.size());
        }
        std::printf("k=%d coverage %.4f hit_rate %.4f multi %.0f\n", k, n_multi ? cov / n_multi : 0.0,
                    others ? hits / others : 0.0, n_multi);
    }
    return 0;
}
'''


def test_slot_policy(tmp_path):
    src = os.path.join(tmp_path, "driver.cpp")
    exe = os.path.join(tmp_path, "driver")
    with open(src, "w") as f:
        f.write(DRIVER)
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", B.CSRC, src, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr


FAKE = 0x10000
OK, INVALID, UNSUPPORTED = 0, 1, 2


def test_pool_manager_host_checks():
    B.build()
    lib = L.load()
    h = ctypes.c_void_p()

    def storage(**kw):
        d = dict(A=FAKE, B=FAKE, A_off=FAKE, B_off=FAKE, rank=FAKE, A_elems=8 * 16 * 64, B_elems=8 * 32 * 16,
                 n_adapters=8, d_in=64, d_out=32, max_rank=16)
        d.update(kw)
        return L.LoraPoolStruct(**d)

    assert lib.lora_pm_create(ctypes.byref(storage(A=0)), None, ctypes.byref(h)) == INVALID
    assert lib.lora_pm_create(ctypes.byref(storage(A_elems=100)), None, ctypes.byref(h)) == INVALID
    assert lib.lora_pm_create(ctypes.byref(storage(max_rank=12)), None, ctypes.byref(h)) == UNSUPPORTED
    assert lib.lora_pm_create(ctypes.byref(storage(d_in=60)), None, ctypes.byref(h)) == UNSUPPORTED
    assert lib.lora_pm_create(None, None, ctypes.byref(h)) == INVALID
    assert lib.lora_pm_register(None, 1, FAKE, FAKE, 16) == INVALID
    assert lib.lora_pm_acquire(None, FAKE, 1, None, None, None) == INVALID


def test_cooccurrence_preloading_coverage(tmp_path):
    """Top-k co-occurrence preloading on a synthetic stream of 1-3-adapter requests with
    recurring combinations (workloads.cooccurrence_requests): coverage grows with k, most
    of a multi-adapter request's companions are predicted at k = 3, and preloading raises
    the share of companions already resident when they are needed."""
    from workloads import cooccurrence_requests
    reqs = cooccurrence_requests(seed=4, n_requests=20000)
    stream = tmp_path / "requests.txt"
    stream.write_text("\n".join(" ".join(str(int(a)) for a in r) for r in reqs) + "\n")
    src = tmp_path / "cov.cpp"
    exe = tmp_path / "cov"
    src.write_text(COVERAGE_DRIVER)
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-I", B.CSRC, str(src), "-o", str(exe)])
    out = subprocess.run([str(exe), str(stream)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    rows = {}
    for line in out.stdout.split("\n"):
        if line.startswith("k="):
            f = line.split()
            rows[int(f[0][2:])] = (float(f[2]), float(f[4]))
    print(out.stdout)
    cov = [rows[k][0] for k in range(4)]
    hit = [rows[k][1] for k in range(4)]
    assert cov[0] == 0.0 and cov[1] <= cov[2] <= cov[3]
    assert cov[3] > 0.6
    assert hit[3] > hit[0] + 0.2
