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
    std::printf("fails %d\n", fails);
    return fails != 0;
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
