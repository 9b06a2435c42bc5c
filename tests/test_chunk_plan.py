"""The row partition every merge kernel uses (ChunkPlan in rowcombine.cuh) and
the merge grid size (merge_grid), compiled for the host with nvcc and checked
on the CPU: every output row belongs to exactly one warp's chunk, chunks hold
1..32 rows, full rounds give neighbouring warps neighbouring chunks, and the
rows left after them are split evenly (no warp more than one row-slice
behind another). No GPU is needed: the code under test is host-callable."""
from __future__ import annotations

import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "lse_pack_stable_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

PROGRAM = r'''
#include <cstdio>
#include <vector>
#include "rowcombine.cuh"
namespace cplse { int sm_count() { return 148; } }
using namespace cplse;

static int check(int64_t rows, int64_t nwarps) {
    std::vector<int> cover(rows, 0);
    int64_t min_rows = -1, max_rows = 0;
    for (int64_t w = 0; w < nwarps; ++w) {
        const ChunkPlan p(rows, w, nwarps);
        int64_t mine = 0;
        for (int64_t i = 0; i < p.count(); ++i) {
            int64_t start; int n;
            p.chunk(i, start, n);
            if (n < 1 || n > 32 || start < 0 || start + n > rows) return 1;
            if (i < p.full && start != (w + i * nwarps) * 32) return 2;
            for (int64_t q = start; q < start + n; ++q) cover[q]++;
            mine += n;
        }
        if (min_rows < 0 || mine < min_rows) min_rows = mine;
        if (mine > max_rows) max_rows = mine;
    }
    for (int64_t q = 0; q < rows; ++q) if (cover[q] != 1) return 3;
    // the last round is split evenly: at most one slice (<= 32 rows) apart
    if (max_rows - min_rows > 32) return 4;
    return 0;
}

int main() {
    const int64_t rows[] = {1, 7, 31, 32, 33, 100, 1000, 4095, 4097, 32768, 131072, 1048576};
    const int64_t warps[] = {1, 2, 3, 4, 37, 128, 1184, 2368, 4144};
    for (int64_t r : rows)
        for (int64_t w : warps) {
            if (r * w > (int64_t)1 << 31) continue;
            const int e = check(r, w);
            if (e) { std::printf("FAIL rows=%lld warps=%lld code=%d\n", (long long)r, (long long)w, e); return 1; }
        }
    // merge_grid: at least one block, at most the resident blocks, and enough warps
    // for min_rows rows each when the GPU has room
    if (merge_grid(1, 128, 7, 4) != 1) return 5;
    if (merge_grid(131072, 128, 7, 4) != 7 * 148) return 6;
    if (merge_grid(32768, 128, 8, 4) != 8 * 148) return 7;
    if (merge_grid(64, 128, 8, 4) != 4) return 8;      // 16 warps of 4 rows: 4 blocks of 4 warps
    std::printf("OK\n");
    return 0;
}
'''


@pytest.mark.skipif(not os.path.exists(NVCC) and shutil.which("nvcc") is None, reason="needs nvcc")
def test_chunk_plan_covers_every_row_once():
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "plan.cu")
        exe = os.path.join(d, "plan")
        with open(src, "w") as f:
            f.write(PROGRAM)
        r = subprocess.run([nvcc, "-std=c++17", "-O1", "-I" + CSRC,
                            "-I" + os.path.join(ROOT, "include"), src, "-o", exe],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-3000:]
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0 and out.stdout.strip() == "OK", out.stdout + out.stderr
