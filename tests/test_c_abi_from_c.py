"""The boundary from plain C: include/absp.h compiles as C99 with warnings
as errors, and a C program linked against libabsp.so makes the host-only
calls (status strings, size queries, argument checks) with the results the
layout fixes.  No device work is launched."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "absp.h"

#define CHECK(c) do { if (!(c)) { printf("FAIL line %d: %s\n", __LINE__, #c); return 1; } } while (0)

int main(void) {
    /* fake, never dereferenced device addresses (256-byte aligned) */
    int32_t bs[2] = {16, 64};
    absp_layer_kv kv;
    memset(&kv, 0, sizeof kv);
    kv.num_seqs = 1;
    kv.num_q_heads = 8;
    kv.num_kv_heads = 2;
    kv.head_dim = ABSP_HEAD_DIM;
    kv.page_size = ABSP_PAGE_SIZE;
    kv.max_pages_per_seq = 512;
    kv.num_phys_pages = 512;
    kv.seq_lens = (const int32_t*)0x10000;
    kv.page_table = (const int32_t*)0x20000;
    kv.k_pages = (const void*)0x100000;
    kv.v_pages = (const void*)0x200000;
    kv.block_size = bs;

    size_t codes = 0, scale = 0, zp = 0, ws = 0;
    CHECK(absp_centroid_sizes(&kv, &codes, &scale, &zp) == ABSP_OK);
    CHECK(codes == (512 + 128) * ABSP_CODE_ROW_BYTES);      /* 8192 tokens at 16 and 64 */
    CHECK(scale == 2 * 128 * 4 && zp == 2 * 128 * 4);
    int64_t row = -1;
    CHECK(absp_centroid_row_offset(&kv, 0, 1, &row) == ABSP_OK && row == 512);
    int32_t kmax = 0;
    CHECK(absp_select_capacity(&kv, 1024, &kmax) == ABSP_OK && kmax == 64);
    CHECK(absp_build_workspace_size(&kv, &ws) == ABSP_OK && ws > 0);
    CHECK(absp_decode_workspace_size(&kv, 1024, &ws) == ABSP_OK && ws > 0);

    /* argument errors come back as statuses, before any device work */
    CHECK(absp_select_capacity(&kv, 8, &kmax) == ABSP_ERR_INVALID_ARG);
    kv.head_dim = 64;
    CHECK(absp_centroid_sizes(&kv, &codes, &scale, &zp) == ABSP_ERR_UNSUPPORTED);
    kv.head_dim = ABSP_HEAD_DIM;
    CHECK(absp_decode_step_ex(&kv, NULL, NULL, 1024, NULL, NULL, 0, 0x80u, NULL) ==
          ABSP_ERR_INVALID_ARG);
    CHECK(absp_build_centroids(&kv, (void*)0x400000, 64, NULL) == ABSP_ERR_INVALID_ARG);
    CHECK(absp_centroid_sizes(NULL, NULL, NULL, NULL) == ABSP_ERR_INVALID_ARG);

    CHECK(strcmp(absp_status_string(ABSP_OK), "ok") == 0);
    CHECK(strcmp(absp_status_string(99), "unknown status") == 0);
    CHECK(absp_last_cuda_error() == 0);
    CHECK(absp_last_cuda_error_string() != NULL);
    printf("ok\n");
    return 0;
}
"""


@pytest.fixture(scope="module")
def lib_path():
    from block_sparse_attention_kv_b200 import build
    return build.build()


def test_header_is_c99_and_the_library_links_from_c(lib_path, tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_absp.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_absp"
    libdir = os.path.dirname(lib_path)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-labsp", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
