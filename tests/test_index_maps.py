"""Host-side check of the kernels' index helpers (csrc/internal.h), compiled for the CPU.

HeadRef maps (batch b, head hh, position i) of a [B, heads, L, 64] tensor held in either memory
layout to its memory row and to the coordinates of the tile maps; kv_head_of maps a query head to
its key/value head.  Both are compared here with what torch's strides and the grouped-query head
rule give, without a GPU: a small host program includes the header and prints its answers.
"""
import shutil
import subprocess
from pathlib import Path

import pytest
import torch

ROOT = Path(__file__).resolve().parents[1]
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

PROGRAM = r"""
#include <cstdio>
#include <cstdlib>
#include "internal.h"
using namespace entmax;
int main(int argc, char** argv) {
    const int layout = atoi(argv[1]), B = atoi(argv[2]), nh = atoi(argv[3]), L = atoi(argv[4]);
    const int H = atoi(argv[5]), Hkv = atoi(argv[6]);
    for (int b = 0; b < B; ++b)
        for (int hh = 0; hh < nh; ++hh) {
            const HeadRef r{layout, b, hh, nh, L};
            for (int i = 0; i < L; ++i)
                printf("R %d %d %d %zu %d %d %zu\n", b, hh, i, r.row(i), r.c1(i), r.c2(i), r.row(0) + i * r.step());
        }
    for (int bh = 0; bh < B * H; ++bh) printf("K %d %d\n", bh, kv_head_of(bh, H, Hkv));
    return 0;
}
"""


@pytest.fixture(scope="module")
def index_program(tmp_path_factory):
    if not Path(NVCC).exists():
        pytest.skip("needs nvcc")
    d = tmp_path_factory.mktemp("index_maps")
    src = d / "index_maps.cu"
    src.write_text(PROGRAM)
    exe = d / "index_maps"
    cmd = [NVCC, "-std=c++17", "-I", str(ROOT / "entmax_tcgen05_tma_b200" / "csrc"), "-I", str(ROOT / "include"),
           str(src), "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    return exe


def _run(exe, *args):
    r = subprocess.run([str(exe), *map(str, args)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    rows, kv = [], []
    for ln in r.stdout.splitlines():
        f = ln.split()
        (rows if f[0] == "R" else kv).append(tuple(int(x) for x in f[1:]))
    return rows, kv


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("B,nh,L", [(3, 5, 7), (2, 1, 130), (1, 4, 1)])
def test_head_rows_and_tile_coordinates(index_program, layout, B, nh, L):
    rows, _ = _run(index_program, layout, B, nh, L, nh, nh)
    assert len(rows) == B * nh * L
    # the [B, heads, L, 64] view the binding passes: contiguous, or a transpose(1, 2) of [B, L, heads, 64]
    x = torch.empty(B, nh, L, 64) if layout == 0 else torch.empty(B, L, nh, 64).transpose(1, 2)
    s0, s1, s2, s3 = x.stride()
    assert s3 == 1
    # tile-map geometry: dims (64, L, B*heads) for layout 0 and (64, heads, B*L) for layout 1,
    # coordinates (0, c1, c2); outer strides in elements
    m1, m2 = (64, 64 * L) if layout == 0 else (64, 64 * nh)
    for b, hh, i, row, c1, c2, stepped in rows:
        off = b * s0 + hh * s1 + i * s2
        assert row * 64 == off
        assert stepped == row
        assert c1 * m1 + c2 * m2 == off
        assert 0 <= c1 < (L if layout == 0 else nh) and 0 <= c2 < (B * nh if layout == 0 else B * L)


@pytest.mark.parametrize("B,H,Hkv", [(2, 8, 2), (3, 6, 3), (1, 4, 1), (2, 5, 5), (4, 32, 8)])
def test_kv_head_of_follows_the_group_rule(index_program, B, H, Hkv):
    _, kv = _run(index_program, 0, B, 1, 1, H, Hkv)
    assert len(kv) == B * H
    for bh, g in kv:
        b, h = divmod(bh, H)
        assert g == b * Hkv + h // (H // Hkv)
