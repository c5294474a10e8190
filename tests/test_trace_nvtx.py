"""Per-call tracing: every C-ABI call that queues device work opens an NVTX
range named "pkv:<call>" for the duration of the call.

Checked on the CPU with a stand-in profiler: a small NVTX injection library
(compiled here with gcc) that records each range push and pop into a file.
NVTX loads it through NVTX_INJECTION64_PATH at the first range, exactly as a
real tool would be loaded.  The calls are made on a host-only pool, so each
returns INVALID_ARG after opening its range; no GPU is involved.
"""

import os
import subprocess
import sys
import textwrap

import pytest

import pagedattention_decode_02_b200 as pk

INJECTION_C = r"""
#include <stdio.h>
#include <stdlib.h>
#include <nvtx3/nvToolsExt.h>

static FILE* g_log;
static int NVTX_API push_a(const char* name) { fprintf(g_log, "push %s\n", name); fflush(g_log); return 0; }
static int NVTX_API pop(void) { fprintf(g_log, "pop\n"); fflush(g_log); return 0; }

int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
    g_log = fopen(getenv("PKV_NVTX_LOG"), "w");
    if (!g_log) return 0;
    const NvtxExportTableCallbacks* cb =
        (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
    NvtxFunctionTable table = 0;
    unsigned int n = 0;
    if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &n)) return 0;
    if (n <= NVTX_CBID_CORE_RangePop) return 0;
    *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)push_a;
    *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)pop;
    return 1;
}
"""

CALLS = textwrap.dedent(r"""
    import ctypes, sys
    lib = ctypes.CDLL(sys.argv[1])
    P = ctypes.c_void_p
    pool = P()
    assert lib.kv_pool_create(4, 16, 1, 64, 1, ctypes.c_float(1), ctypes.c_float(1), None, None,
                              1, None, ctypes.byref(pool)) == 0
    one = (ctypes.c_int32 * 4)()
    lib.kv_append(pool, one, 1, one, one, 1, None)
    lib.block_copy(pool, one, one, 1, None)
    lib.paged_decode_attention(pool, one, 1, one, 1, one, 1, 1, ctypes.c_float(1.0), one, None,
                               ctypes.c_size_t(0), None)
    lib.paged_decode_attention_static(pool, one, 1, one, 1, one, 1, 1, ctypes.c_float(1.0), one,
                                      0, None)
    lib.paged_prefill_attention(pool, one, 1, one, 1, one, 1, one, 1, 1, ctypes.c_float(1.0), one,
                                None)
    n_blocks = ctypes.c_int32()
    n_tok = ctypes.c_int64()
    lib.kv_swap_out(pool, ctypes.c_int64(0), one, one, ctypes.c_size_t(16), ctypes.byref(n_blocks),
                    ctypes.byref(n_tok), None)
    lib.kv_swap_in(pool, ctypes.c_int64(0), one, one, ctypes.c_size_t(16), ctypes.c_int64(1), None)
    lib.kv_pool_destroy(pool)
""")


def test_device_calls_open_named_ranges(tmp_path):
    so = tmp_path / "libfaketool.so"
    src = tmp_path / "faketool.c"
    src.write_text(INJECTION_C)
    r = subprocess.run(["gcc", "-shared", "-fPIC", "-O1", "-I/usr/local/cuda/include", str(src),
                        "-o", str(so)], capture_output=True, text=True)
    if r.returncode != 0:
        pytest.skip("no gcc / NVTX headers: " + r.stderr[-300:])
    log = tmp_path / "ranges.log"
    env = dict(os.environ, NVTX_INJECTION64_PATH=str(so), PKV_NVTX_LOG=str(log))
    r = subprocess.run([sys.executable, "-c", CALLS, pk.LIB_PATH], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    lines = log.read_text().splitlines()
    pushed = [ln[5:] for ln in lines if ln.startswith("push ")]
    for want in ("kv_append", "block_copy", "paged_decode_attention_ex",
                 "paged_decode_attention_static", "paged_prefill_attention_ex", "kv_swap_out",
                 "kv_swap_in"):
        assert "pkv:" + want in pushed, (want, pushed)
    # every range that opened was closed, in nesting order
    depth = 0
    for ln in lines:
        depth += 1 if ln.startswith("push ") else -1
        assert depth >= 0
    assert depth == 0
