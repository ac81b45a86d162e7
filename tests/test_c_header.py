"""The boundary is a C ABI: include/milo.h compiles as plain C (C99 and C11,
warnings as errors) and a C program links against libmilo.so and calls its
host-side entry points (no GPU: only calls that return before any device
work)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "milo.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void) {
    size_t bytes = 0;
    CHECK(milo_version() >= 1);
    CHECK(strcmp(milo_status_str(MILO_OK), "ok") == 0);
    /* the blob of a [4096, 14336] weight: 64 tiles x 112 super-blocks x 3584 bytes */
    CHECK(milo_packed_bytes(4096, 14336, &bytes) == MILO_OK);
    CHECK(bytes == (size_t)64 * 112 * 3584);
    CHECK(milo_packed_bytes(4096, 100, &bytes) == MILO_ERR_UNSUPPORTED_SHAPE);
    CHECK(strstr(milo_last_error(), "128") != NULL);
    CHECK(milo_table_bytes(3, &bytes) == MILO_OK && bytes > 0);

    /* a layer struct filled by hand: size queries need no device */
    milo_moe_layer layer;
    memset(&layer, 0, sizeof(layer));
    layer.hidden = 4096; layer.inter = 14336; layer.n_routed = 8; layer.n_shared = 0;
    layer.top_k = 2; layer.group = MILO_GROUP; layer.max_rank = 64;
    size_t small = 0, large = 0;
    CHECK(milo_moe_workspace_bytes(&layer, 16, &small) == MILO_OK);
    CHECK(milo_moe_workspace_bytes(&layer, 8192, &large) == MILO_OK);
    CHECK(0 < small && small < large);
    CHECK(milo_moe_h_offset(&layer, 16) % 256 == 0);
    layer.top_k = 9;      /* more than n_routed */
    CHECK(milo_moe_workspace_bytes(&layer, 16, &small) == MILO_ERR_UNSUPPORTED_SHAPE);

    milo_linear lin;
    memset(&lin, 0, sizeof(lin));
    lin.N = 14336; lin.K = 4096; lin.n_experts = 8; lin.group = MILO_GROUP;
    CHECK(milo_linear_workspace_bytes(&lin, 1, 1, &bytes) == MILO_OK);
    CHECK(milo_linear_workspace_bytes(&lin, MILO_MAX_ROWS / 2 + 1, 2, &bytes) == MILO_ERR_UNSUPPORTED_SHAPE);

    /* arguments refused before any launch */
    CHECK(milo_route(NULL, 4, 300, 2, 0, NULL, NULL, NULL, NULL, NULL, NULL, NULL) ==
          MILO_ERR_UNSUPPORTED_SHAPE);
    CHECK(milo_set_gemm_path(7) == MILO_ERR_INVALID_ARG);

    double score[4] = {3.0, 5.0, 3.0, 9.0};
    int32_t ranks[4];
    CHECK(milo_assign_ranks(score, 4, 16, 64, ranks) == MILO_OK);
    CHECK(ranks[0] + ranks[1] + ranks[2] + ranks[3] <= 64);
    CHECK(ranks[3] >= ranks[1] && ranks[1] >= ranks[0] && ranks[0] == ranks[2]);
    printf("ok\n");
    return 0;
}
"""


@pytest.fixture(scope="module")
def libdir():
    from int3_gemm_rank_b200 import build
    build.build()
    return os.path.join(ROOT, "int3_gemm_rank_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
@pytest.mark.parametrize("std", ["c99", "c11"])
def test_header_compiles_as_c_and_links(tmp_path, libdir, std):
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / f"abi_{std}"
    cmd = ["gcc", f"-std={std}", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-L", libdir, "-lmilo", f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
