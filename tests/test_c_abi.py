"""The boundary is a C ABI: a C11 program that includes include/df11.h and
include/nf12.h,
links libdf11.so and calls the host-side entry points (no CUDA call is made).

The program builds the code of a small histogram whose optimal lengths are
fixed by hand (counts 8, 4, 2, 1, 1 -> lengths 1, 2, 3, 4, 4: a dyadic
distribution, so the code is the textbook one), derives the decode tables,
plans the container and checks a status string and an argument error.
"""
import os
import subprocess
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "lossless_bf16_weight_huffman_b200")

C_PROGRAM = textwrap.dedent(r"""
    #include <stdio.h>
    #include <string.h>
    #include "df11.h"
    #include "nf12.h"

    int main(void) {
        uint64_t hist[256];
        memset(hist, 0, sizeof hist);
        hist[120] = 8; hist[121] = 4; hist[122] = 2; hist[123] = 1; hist[124] = 1;
        df_code code;
        if (df_build_code(hist, 32, &code) != DF_OK) return 1;
        const uint8_t want_len[5] = {1, 2, 3, 4, 4};
        const uint32_t want_code[5] = {0x0, 0x2, 0x6, 0xE, 0xF};  /* canonical: 0, 10, 110, 1110, 1111 */
        for (int i = 0; i < 5; ++i) {
            if (code.lengths[120 + i] != want_len[i]) return 2;
            if (code.codes[120 + i] != want_code[i]) return 3;
        }
        if (code.n_symbols != 5 || code.min_len != 1 || code.lengths[0] != 0) return 4;
        size_t words = df_lut_words(&code);
        if (words == 0 || words > 65536) return 5;
        static uint32_t lut[65536];
        if (df_build_lut(&code, lut, words) != DF_OK) return 6;
        df_sizes z;
        if (df_plan(&code, hist, 16, 32, 256, &z) != DF_OK) return 7;
        if (z.total_bits != 8 * 1 + 4 * 2 + 2 * 3 + 1 * 4 + 1 * 4) return 8;
        if (df_plan(&code, hist, 17, 32, 256, &z) != DF_ERR_INVALID_ARG) return 9;  /* total != n */
        df_nf12_sizes nz;
        if (df_nf12_sizes_for(17, &nz) != DF_OK) return 11;
        if (nz.groups != 3 || nz.slots_bytes != 36 || nz.bitmap_bytes != 4 || nz.tiles != 1) return 12;
        if (df_nf12_sizes_for(17, NULL) != DF_ERR_INVALID_ARG) return 13;
        const char* s = df_status_string(DF_ERR_CORRUPT);
        if (!s || !s[0]) return 10;
        printf("c abi ok: %u symbols, %zu table words, %llu bits\n", code.n_symbols, words,
               (unsigned long long)z.total_bits);
        return 0;
    }
""")


@pytest.fixture(scope="module")
def libdir():
    from lossless_bf16_weight_huffman_b200 import build

    build.build_native()
    return PKG


def test_header_compiles_as_c11(tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "df11.h"\n#include "nf12.h"\nint main(void) { return DF_OK; }\n')
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only",
                           "-I", os.path.join(ROOT, "include"), str(src)])


def test_c_program_calls_the_host_entry_points(tmp_path, libdir):
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(C_PROGRAM)
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-o", str(exe), str(src),
                           "-I", os.path.join(ROOT, "include"), "-L", libdir, "-ldf11",
                           "-Wl,-rpath," + libdir])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "c abi ok: 5 symbols" in r.stdout
