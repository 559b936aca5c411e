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
    // segmentation: at least one segment, never more than the chunks, contiguous cover
    CHECK(kda::seg_count(0, 4) == 1 && kda::seg_count(1, 4) == 1 && kda::seg_count(3, 4) == 3);
    CHECK(kda::seg_count(100, 4) == 4 && kda::seg_count(100, 1) == 1);
    for (int chunks = 1; chunks < 300; ++chunks)
        for (int segs = 1; segs < 12; ++segs) {
            const int G = kda::seg_count(chunks, segs);
            CHECK(kda::seg_chunk_begin(chunks, G, 0) == 0 && kda::seg_chunk_begin(chunks, G, G) == chunks);
            for (int g = 0; g < G; ++g) {
                const int len = kda::seg_chunk_begin(chunks, G, g + 1) - kda::seg_chunk_begin(chunks, G, g);
                CHECK(len >= 1 && len <= (chunks + G - 1) / G);
            }
        }
    // totals over a ragged pack: 2500 (40 chunks, 3 segments), 1, 0, 700 (11 chunks), 129 (3)
    const int cu[6] = {0, 2500, 2501, 2501, 3201, 3330};
    const kda::SegTotals t = kda::seg_totals(cu, 5, 3);
    CHECK(t.num_vseqs == 3 + 1 + 1 + 3 + 3);
    CHECK(t.e_chunks == (40 - 13) + (11 - 3) + (3 - 1));
    CHECK(t.max_chunks == 14);
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
