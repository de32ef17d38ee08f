"""The boundary from plain C: include/sbl.h compiles as strict C99 and a C
program linked against the in-tree libsbl.so calls it (no Python, no torch
types).  Only host-side paths run (version, status strings, zero-size no-ops,
argument checks), so no GPU is needed."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "sparse_linear_layers_b200")

PROGRAM = r"""
#include <stdint.h>
#include <stdio.h>
#include "sbl.h"

typedef void (*any_fn)(void);
/* the address of every entry point the header declares: each declaration is
   type-checked by the compiler and resolved by the linker */
static const any_fn entry_points[] = { %(table)s };

#define EXPECT(expr, code)                                                        \
    do {                                                                          \
        int r_ = (int)(expr);                                                     \
        if (r_ != (int)(code)) {                                                  \
            fprintf(stderr, "line %%d: %%s returned %%d, expected %%d\n", __LINE__, \
                    #expr, r_, (int)(code));                                      \
            return 1;                                                             \
        }                                                                         \
    } while (0)

int main(void) {
    /* a fake, 256-byte aligned device address: every call below fails (or
       returns) on the host before any pointer is used */
    void* p = (void*)(uintptr_t)4096;
    const char* v = sbl_version();
    if (!v || !v[0]) return 2;
    if (!sbl_status_string(SBL_ERR_WORKSPACE) || !sbl_status_string(SBL_OK)) return 3;

    /* zero sizes enqueue nothing */
    EXPECT(sbl_quant_act(NULL, 0, 64, NULL, NULL, NULL), SBL_OK);
    EXPECT(sbl_linear(NULL, 0, 64, NULL, NULL, 16, 2, 4, NULL, SBL_F32, NULL, NULL, 0, NULL), SBL_OK);
    EXPECT(sbl_linear_q(NULL, NULL, 4, 64, NULL, NULL, 0, 2, 4, NULL, SBL_F32, NULL, NULL, 0, NULL), SBL_OK);

    /* argument errors, returned synchronously */
    EXPECT(sbl_linear((const uint16_t*)p, 4, 64, (const uint8_t*)p, (const float*)p, 16, 2, 4, p, 7, NULL, p,
                      (size_t)1 << 20, NULL), SBL_ERR_INVALID_ARG);
    EXPECT(sbl_linear((const uint16_t*)p, 4, 64, (const uint8_t*)p, (const float*)p, 16, 2, 4, p, SBL_F32, NULL,
                      p, 16, NULL), SBL_ERR_WORKSPACE);
    EXPECT(sbl_linear_q((const int8_t*)p, (const float*)p, 4, 48, (const uint8_t*)p, (const float*)p, 16, 2, 4, p,
                        SBL_F32, NULL, p, (size_t)1 << 20, NULL), SBL_ERR_UNSUPPORTED);
    EXPECT(sbl_linear_q((const int8_t*)p, (const float*)p, 4, 64, (const uint8_t*)p, (const float*)p, 16, 2, 4, p,
                        SBL_F32, NULL, NULL, (size_t)1 << 20, NULL), SBL_ERR_WORKSPACE);
    EXPECT(sbl_prepare_weights((const float*)p, 16, 64, 1, 4, (uint8_t*)p, (float*)p, NULL, NULL),
           SBL_ERR_UNSUPPORTED);
    EXPECT(sbl_linear_plan(0, 64, 16, 2, 4, (size_t)1 << 20), -SBL_ERR_INVALID_ARG);

    printf("%%s %%u\n", v, (unsigned)(sizeof entry_points / sizeof entry_points[0]));
    return 0;
}
"""


def _declared():
    src = open(os.path.join(INCLUDE, "sbl.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sbl_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def gcc():
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(os.path.join(LIBDIR, "libsbl.so")):
        pytest.skip("libsbl.so not built")
    return cc


def test_header_is_strict_c99(gcc, tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "sbl.h"\n')
    subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", INCLUDE,
                    str(src)], check=True)


def test_c_program_links_and_calls_the_library(gcc, tmp_path):
    names = _declared()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM % {"table": ", ".join(f"(any_fn){n}" for n in names)})
    exe = tmp_path / "abi"
    subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, str(src), "-o",
                    str(exe), "-L", LIBDIR, "-lsbl", f"-Wl,-rpath,{LIBDIR}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    version, count = r.stdout.strip().rsplit(" ", 1)
    assert int(count) == len(names)
