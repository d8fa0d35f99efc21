"""The boundary is a C library: a C11 program that includes include/entmax_attn.h (no C++, no torch)
compiles with warnings as errors, links against the in-tree libentmax_attn.so and calls its
host-side functions.  Only calls that return before reaching the CUDA runtime are made (status
strings, version, workspace size, argument checks with fake device addresses that are never
dereferenced), so this runs without a GPU."""
import shutil
import subprocess
from pathlib import Path

import pytest

import entmax_tcgen05_tma_b200 as E

ROOT = Path(__file__).resolve().parents[1]
CUDA_INC = Path("/usr/local/cuda/include")

PROGRAM = r"""
#include "entmax_attn.h"
#include <stdio.h>
#include <string.h>

#define FAKE ((void*)(uintptr_t)0x10000) /* 16-byte aligned, never dereferenced */

static int fails = 0;
#define EXPECT(c) do { if (!(c)) { printf("FAIL line %d: %s\n", __LINE__, #c); ++fails; } } while (0)

int main(void) {
    const int codes[6] = {ENTMAX_OK, ENTMAX_ERR_ARG, ENTMAX_ERR_UNSUPPORTED, ENTMAX_ERR_CUDA,
                          ENTMAX_ERR_TIMEOUT, ENTMAX_ERR_WORKSPACE};
    for (int i = 0; i < 6; ++i)
        for (int j = 0; j < i; ++j)
            EXPECT(strcmp(entmax_attn_strerror(codes[i]), entmax_attn_strerror(codes[j])) != 0);
    EXPECT(strcmp(entmax_attn_strerror(ENTMAX_OK), "ok") == 0);
    EXPECT(entmax_attn_version() >= 100);

    EXPECT(entmax_attn_bwd_workspace_size(0, 12, 128, 64) == 0);
    size_t ws = entmax_attn_bwd_workspace_size(4, 12, 4096, 64);
    EXPECT(ws >= (size_t)4 * 12 * 4096 * sizeof(float) && ws % 256 == 0);

    float* tau = (float*)FAKE;
    /* head dimension other than 64 */
    EXPECT(entmax_attn_fwd(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.125f, 1, 1, 64, 32, FAKE,
                           ENTMAX_BF16, tau, (cudaStream_t)0) == ENTMAX_ERR_UNSUPPORTED);
    /* null output, non-positive scale, unknown dtype */
    EXPECT(entmax_attn_fwd(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.125f, 1, 1, 64, 64, NULL,
                           ENTMAX_BF16, tau, (cudaStream_t)0) == ENTMAX_ERR_ARG);
    EXPECT(entmax_attn_fwd(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.0f, 1, 1, 64, 64, FAKE,
                           ENTMAX_BF16, tau, (cudaStream_t)0) == ENTMAX_ERR_ARG);
    EXPECT(entmax_attn_fwd(FAKE, FAKE, FAKE, 7, NULL, 0, 0, 0.125f, 1, 1, 64, 64, FAKE,
                           ENTMAX_BF16, tau, (cudaStream_t)0) == ENTMAX_ERR_ARG);
    /* a sliding window needs causal masking */
    EXPECT(entmax_attn_fwd(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 16, 0.125f, 1, 1, 64, 64, FAKE,
                           ENTMAX_BF16, tau, (cudaStream_t)0) == ENTMAX_ERR_UNSUPPORTED);
    /* backward without its workspace */
    EXPECT(entmax_attn_bwd(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.125f, 1, 1, 64, 64, tau, FAKE,
                           (float*)FAKE, (float*)FAKE, (float*)FAKE, NULL, 0, (cudaStream_t)0)
           == ENTMAX_ERR_WORKSPACE);
    /* alpha below 1 (the softmax band is |alpha - 1| < 1e-4) or above 2 is a bad argument */
    EXPECT(entmax_attn_fwd_ex(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.125f, 0.999f, 1, 2, 1, 64, 64,
                              ENTMAX_LAYOUT_BHLD, FAKE, ENTMAX_BF16, tau, NULL, 0, (cudaStream_t)0)
           == ENTMAX_ERR_ARG);
    EXPECT(entmax_attn_fwd_ex(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.125f, 2.5f, 1, 2, 1, 64, 64,
                              ENTMAX_LAYOUT_BHLD, FAKE, ENTMAX_BF16, tau, NULL, 0, (cudaStream_t)0)
           == ENTMAX_ERR_ARG);
    /* key/value heads that do not divide the query heads */
    EXPECT(entmax_attn_fwd_gqa(FAKE, FAKE, FAKE, ENTMAX_BF16, NULL, 0, 0, 0.125f, 1, 4, 3, 64, 64, FAKE,
                               ENTMAX_BF16, tau, (cudaStream_t)0) == ENTMAX_ERR_ARG);
    printf("%d failures\n", fails);
    return fails != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None or not CUDA_INC.is_dir(), reason="needs gcc and the CUDA headers")
def test_c_program_against_the_header_and_library(tmp_path):
    src = tmp_path / "client.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "client"
    lib_dir = Path(E.LIB_PATH).parent
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", str(ROOT / "include"), "-I", str(CUDA_INC),
           str(src), "-L", str(lib_dir), "-lentmax_attn", "-Wl,-rpath," + str(lib_dir), "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 failures" in r.stdout
