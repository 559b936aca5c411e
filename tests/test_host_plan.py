"""Host-side bookkeeping of the library, unit-tested on the CPU with g++ (no GPU, no CUDA types).

csrc/host_plan.h holds (1) PerDeviceOnce, the once-per-device guard behind each kernel's
dynamic shared-memory limit (a per-context attribute: a process-wide flag would skip the set-up
on the second GPU a process uses), and (2) split_coresident, the check that decides whether the
split-role prefill's cooperative launch fits on this device or the single-role kernel runs.
"""
import os
import subprocess
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_62_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <thread>
#include <vector>
#include "host_plan.h"

#define CHECK(c) do { if (!(c)) { std::printf("FAIL line %d: %s\n", __LINE__, #c); return 1; } } while (0)

int main() {
    kda::PerDeviceOnce<8> once;
    int calls[8] = {};
    auto setup = [&](int dev, int result) { return once.run(dev, [&] { ++calls[dev]; return result; }); };
    // first device: set up once, never again
    CHECK(setup(0, 0) == 0 && calls[0] == 1);
    CHECK(setup(0, 0) == 0 && calls[0] == 1);
    // a second device still gets its own set-up (the bug a process-wide flag had)
    CHECK(!once.done(1));
    CHECK(setup(1, 0) == 0 && calls[1] == 1 && once.done(1));
    // a failed set-up is reported and retried, not remembered
    CHECK(setup(2, 98) == 98 && calls[2] == 1 && !once.done(2));
    CHECK(setup(2, 0) == 0 && calls[2] == 2 && once.done(2));
    CHECK(setup(2, 98) == 0 && calls[2] == 2);
    // device ids outside the table
    CHECK(once.run(-1, [] { return 0; }) == kda::PerDeviceOnce<8>::kBadDevice);
    CHECK(once.run(8, [] { return 0; }) == kda::PerDeviceOnce<8>::kBadDevice);
    // many threads racing on one device: exactly one set-up
    kda::PerDeviceOnce<8> race;
    int n = 0;
    std::vector<std::thread> ts;
    for (int i = 0; i < 16; ++i) ts.emplace_back([&] { race.run(3, [&] { ++n; return 0; }); });
    for (auto &t : ts) t.join();
    CHECK(n == 1);
    // split co-residency: one block per SM on 148 SMs fits up to 74 heads (a producer per consumer)
    CHECK(kda::split_coresident(1, 148, 37));
    CHECK(kda::split_coresident(1, 148, 74));
    CHECK(!kda::split_coresident(1, 148, 75));
    CHECK(!kda::split_coresident(0, 148, 1));    // the kernel does not fit on an SM at all
    CHECK(!kda::split_coresident(1, 20, 16));    // few SMs visible (a partitioned context)
    CHECK(kda::split_coresident(2, 16, 16));
    CHECK(!kda::split_coresident(1, 148, 0));
    std::printf("ok\n");
    return 0;
}
"""


def test_host_plan_bookkeeping():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "t.cpp")
        exe = os.path.join(d, "t")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, src, "-o", exe], check=True)
        r = subprocess.run([exe], capture_output=True, text=True)
        assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
