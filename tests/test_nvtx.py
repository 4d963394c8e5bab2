"""Every public entry point opens an NVTX range named after itself (host-side, no GPU needed).

A small NVTX injection library, built here with gcc, replaces the push and pop callbacks with
functions that log the range names to a file; a child process loads the library under it and
makes calls that stop in host-side validation.  Each call must log its own push and pop."""
import os
import subprocess
import sys
import textwrap

import pytest

from learned_sparse_kv_b200 import build as lbuild

INJECTION = r"""
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
typedef void (*fn_t)(void);
typedef fn_t **fn_table_t;
typedef struct {
    size_t struct_size;
    int (*get_module_function_table)(int module, fn_table_t *table, unsigned int *size);
} callbacks_t;
typedef const void *(*get_export_table_t)(uint32_t id);
static FILE *log_file;
static int push_a(const char *name) { fprintf(log_file, "push %s\n", name); fflush(log_file); return 0; }
static int pop(void) { fprintf(log_file, "pop\n"); fflush(log_file); return 0; }
/* export table 1: callbacks; module 1: core; slots 9 and 11: RangePushA and RangePop */
int InitializeInjectionNvtx2(get_export_table_t get) {
    const callbacks_t *cb = (const callbacks_t *)get(1);
    fn_table_t table;
    unsigned int size = 0;
    if (!cb || !cb->get_module_function_table(1, &table, &size) || size <= 11) return 0;
    log_file = fopen(getenv("LSA_NVTX_LOG"), "w");
    if (!log_file) return 0;
    *table[9] = (fn_t)push_a;
    *table[11] = (fn_t)pop;
    return 1;
}
"""

CHILD = textwrap.dedent("""
    import ctypes, sys
    lib = ctypes.CDLL(sys.argv[1])
    P = ctypes.c_void_p(4096)
    # both calls stop in host-side validation: nothing is enqueued
    rc1 = lib.lsa_label_vote(P, 65, 4, 128, ctypes.c_float(0.6), 3, 0, P, None, P, ctypes.c_size_t(1 << 20), None)
    rc2 = lib.lsa_advance_window(P, P, 0, 64, 1, None)
    print(rc1, rc2)
""")


@pytest.fixture(scope="module")
def injection(tmp_path_factory):
    d = tmp_path_factory.mktemp("nvtx")
    src = d / "inject.c"
    src.write_text(INJECTION)
    so = d / "libinject.so"
    r = subprocess.run(["gcc", "-shared", "-fPIC", "-O1", "-o", str(so), str(src)], capture_output=True, text=True)
    if r.returncode != 0:
        pytest.skip("gcc could not build the injection library: " + r.stderr[:200])
    return so


def test_entry_points_open_named_nvtx_ranges(injection, tmp_path):
    lib = lbuild.build()
    log = tmp_path / "ranges.log"
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(injection), LSA_NVTX_LOG=str(log))
    r = subprocess.run([sys.executable, "-c", CHILD, lib], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    rc1, rc2 = map(int, r.stdout.split())
    assert rc1 == 2 and rc2 == 1            # shape error, then a bad batch size
    assert log.read_text().split("\n")[:4] == ["push lsa_label_vote", "pop", "push lsa_advance_window", "pop"]
