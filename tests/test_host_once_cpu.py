"""The launchers' per-device, compute-once cache (csrc/host_once.h) under
concurrent host threads, compiled with g++ on the CPU: each device's value is
computed exactly once however many threads ask at the same time, every
thread sees that value, a failed computation is retried, and devices out of
range are refused."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "binary_weight_transformer_b200", "csrc")

PROGRAM = r"""
#include <atomic>
#include <chrono>
#include <cstdio>
#include <thread>
#include <vector>
#include "host_once.h"

int main()
{
    lowbit::PerDevice cache;
    std::atomic<int> calls[3] = {};
    std::atomic<int> wrong{0};
    std::vector<std::thread> threads;
    for (int t = 0; t < 16; ++t) {
        threads.emplace_back([&, t] {
            for (int rep = 0; rep < 1000; ++rep) {
                const int dev = (t + rep) % 3;
                const int v = cache.get(dev, [&] {
                    calls[dev].fetch_add(1);
                    std::this_thread::sleep_for(std::chrono::milliseconds(5));
                    return 100 + dev;
                });
                if (v != 100 + dev) wrong.fetch_add(1);
            }
        });
    }
    for (auto &th : threads) th.join();

    // a failed computation is returned, not kept, and retried
    lowbit::PerDevice retry;
    int attempts = 0;
    const int first = retry.get(5, [&] { ++attempts; return 0; });
    const int second = retry.get(5, [&] { ++attempts; return 7; });
    const int third = retry.get(5, [&] { ++attempts; return 9; });
    // out of range
    const int outside = retry.get(64, [&] { return 1; }) + retry.get(-1, [&] { return 1; });

    std::printf("%d %d %d %d %d %d %d %d %d\n", calls[0].load(), calls[1].load(), calls[2].load(), wrong.load(),
                first, second, third, attempts, outside);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_per_device_cache_computes_once_across_threads(tmp_path):
    src = tmp_path / "once.cpp"
    exe = tmp_path / "once"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O2", "-pthread", "-I", HEADER_DIR, str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=120).stdout.split()
    calls0, calls1, calls2, wrong, first, second, third, attempts, outside = map(int, out)
    assert (calls0, calls1, calls2) == (1, 1, 1)
    assert wrong == 0
    assert (first, second, third, attempts) == (0, 7, 7, 2)
    assert outside == 0
