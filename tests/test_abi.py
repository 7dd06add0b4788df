"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol the public header declares, and rejects invalid arguments on the
host before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ts_verify.h")


@pytest.fixture(scope="module")
def lib():
    from lossless_ultra_long_b200 import build
    build.build()
    import lossless_ultra_long_b200 as L
    return L.library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^TS_API[^(;]*?\b(ts_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_three_calls():
    syms = declared_symbols()
    for name in ("ts_tree_verify_attn", "ts_kv_importance_select", "ts_penalize_accept"):
        assert name in syms


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_binding_export_list_matches_header():
    import lossless_ultra_long_b200 as L
    assert set(L.EXPORTS) <= set(declared_symbols())


def test_status_strings(lib):
    for code in range(7):
        assert lib.ts_status_string(code)
    assert lib.ts_version() >= 100


def _attn_call(lib, **over):
    args = dict(q=1 << 20, k=1 << 20, v=1 << 20, kv_cap=100, hq=8, hkv=2, d=64, n_ctx=50, t=4,
                parent=np.array([-1, 0, 0, 1], np.int32), scale=0.125, out=1 << 20,
                ws=1 << 20, ws_bytes=1 << 30)
    args.update(over)
    P = ctypes.c_void_p
    par = args["parent"]
    return lib.ts_tree_verify_attn(P(args["q"]), P(args["k"]), P(args["v"]), args["kv_cap"],
                                   args["hq"], args["hkv"], args["d"], args["n_ctx"], args["t"],
                                   par.ctypes.data_as(P) if par is not None else None,
                                   args["scale"], P(args["out"]), P(args["ws"]),
                                   args["ws_bytes"], None)


@pytest.mark.parametrize("over,code", [
    (dict(q=0), 1),
    (dict(hq=6, hkv=4), 1),
    (dict(parent=np.array([0, 0, 0, 1], np.int32)), 1),
    (dict(parent=np.array([-1, 0, 2, 1], np.int32)), 1),
    (dict(parent=None), 1),
    (dict(t=65, parent=np.array([-1] + list(range(64)), np.int32)), 1),
    (dict(kv_cap=53), 1),
    (dict(scale=float("nan")), 1),
    (dict(q=(1 << 20) + 8), 1),
    (dict(d=96), 2),
    (dict(ws=0), 3),
    (dict(ws=(1 << 20) + 128), 3),
    (dict(ws_bytes=16), 3),
])
def test_attention_rejects_on_host(lib, over, code):
    assert _attn_call(lib, **over) == code


def test_select_and_penalize_reject_on_host(lib):
    P = ctypes.c_void_p
    a = P(1 << 20)
    # partial_cap smaller than n_sink + budget
    assert lib.ts_kv_importance_select(a, a, a, 1000, 8, 2, 64, 1000, 16, 240, 0.125, None, a, a,
                                       a, 100, a, 1 << 30, None) == 1
    # group larger than supported
    assert lib.ts_kv_importance_select(a, a, a, 1000, 64, 2, 64, 1000, 16, 240, 0.125, None, a, a,
                                       a, 256, a, 1 << 30, None) == 2
    par = np.array([-1, 0], np.int32)
    pp = par.ctypes.data_as(P)
    assert lib.ts_penalize_accept(a, 2, 100, a, 4, ctypes.c_float(0.0), pp, a, None, a, a,
                                  1 << 20, None) == 1
    assert lib.ts_penalize_accept(a, 2, 100, None, 4, ctypes.c_float(1.2), pp, a, None, a, a,
                                  1 << 20, None) == 1
    assert lib.ts_penalize_accept(a, 2, 100, a, 4, ctypes.c_float(1.2), pp, a, None, a, a,
                                  8, None) == 3
    # vocabularies past what one launch covers
    assert lib.ts_penalize_accept(a, 2, (1 << 24) + 1, a, 4, ctypes.c_float(1.2), pp, a, None,
                                  a, a, 1 << 30, None) == 2
    sample = lib.ts_penalize_sample_accept
    sample.restype = ctypes.c_int
    sample.argtypes = [P, P, ctypes.c_float, ctypes.c_int, ctypes.c_int, P, ctypes.c_int,
                       ctypes.c_float, P, P, ctypes.c_uint, ctypes.c_uint64, P, P, P,
                       ctypes.c_size_t, P]
    assert sample(a, a, 1.0, 2, (1 << 23) + 1, a, 4, 1.2, pp, a, 0, 0, None, a, a, 1 << 30,
                  None) == 2
    # no noise, a bad temperature, unknown flags
    assert sample(a, None, 1.0, 2, 100, a, 4, 1.2, pp, a, 0, 0, None, a, a, 1 << 30, None) == 1
    for t in (0.0, -1.0, float("inf"), float("nan")):
        assert sample(a, a, t, 2, 100, a, 4, 1.2, pp, a, 0, 0, None, a, a, 1 << 30, None) == 1
    assert sample(a, a, 1.0, 2, 100, a, 4, 1.2, pp, a, 8, 0, None, a, a, 1 << 30, None) == 1


def test_workspace_sizes_are_positive_and_zero_for_invalid(lib):
    import lossless_ultra_long_b200 as L
    assert L.tree_verify_attn_workspace_size(32, 8, 128, 102400, 40) > 0
    assert L.tree_verify_attn_workspace_size(32, 8, 96, 1024, 40) == 0
    assert L.kv_importance_select_workspace_size(32, 8, 128, 102400) > 0
    assert L.penalize_accept_workspace_size(40, 128256) > 0
    assert L.penalize_accept_workspace_size(0, 128256) == 0


def _root_scores_call(lib, rs=1 << 20, **over):
    args = dict(q=1 << 20, k=1 << 20, v=1 << 20, kv_cap=100, hq=8, hkv=2, d=64, n_ctx=50, t=4,
                parent=np.array([-1, 0, 0, 1], np.int32), scale=0.125, out=1 << 20,
                ws=1 << 20, ws_bytes=1 << 30)
    args.update(over)
    P = ctypes.c_void_p
    return lib.ts_tree_verify_attn_root_scores(
        P(args["q"]), P(args["k"]), P(args["v"]), args["kv_cap"], args["hq"], args["hkv"],
        args["d"], args["n_ctx"], args["t"], args["parent"].ctypes.data_as(P), args["scale"],
        P(args["out"]), P(rs) if rs else None, P(args["ws"]), args["ws_bytes"], None)


@pytest.mark.parametrize("rs,over,code", [
    (0, {}, 1),                          # no scores buffer
    ((1 << 20) + 2, {}, 1),              # scores not 4-byte aligned
    (1 << 20, dict(hq=32, hkv=2), 2),    # group of 16 > TS_MAX_SELECT_GROUP
    (1 << 20, dict(q=0), 1),             # the attention's own checks still apply
    (1 << 20, dict(d=96), 2),
    (1 << 20, dict(ws_bytes=16), 3),
])
def test_root_scores_attention_rejects_on_host(lib, rs, over, code):
    assert _root_scores_call(lib, rs, **over) == code


def _from_scores_call(lib, **over):
    args = dict(rs=1 << 20, k=1 << 20, v=1 << 20, kv_cap=1000, hq=8, hkv=2, d=64, n_ctx=1000,
                n_sink=16, budget=240, scores=None, idx=1 << 20, kp=1 << 20, vp=1 << 20,
                cap=256, ws=1 << 20, ws_bytes=1 << 20)
    args.update(over)
    P = ctypes.c_void_p
    p = lambda x: P(x) if x else None
    return lib.ts_kv_select_from_scores(
        p(args["rs"]), p(args["k"]), p(args["v"]), args["kv_cap"], args["hq"], args["hkv"],
        args["d"], args["n_ctx"], args["n_sink"], args["budget"], p(args["scores"]),
        p(args["idx"]), p(args["kp"]), p(args["vp"]), args["cap"], p(args["ws"]),
        args["ws_bytes"], None)


@pytest.mark.parametrize("over,code", [
    (dict(rs=0), 1),
    (dict(idx=0), 1),
    (dict(cap=255), 1),                  # partial cache shorter than n_sink + budget
    (dict(n_ctx=1001), 1),               # context past the cache capacity
    (dict(n_sink=-1), 1),
    (dict(rs=(1 << 20) + 4), 1),         # n_ctx % 4 == 0: rows read 16 bytes at a time
    (dict(rs=(1 << 20) + 2), 1),
    (dict(kp=(1 << 20) + 8), 1),
    (dict(hq=6, hkv=4), 1),
    (dict(hq=64, hkv=2), 2),             # group of 32
    (dict(d=96), 2),
    (dict(ws=0), 3),
    (dict(ws_bytes=8), 3),
])
def test_select_from_scores_rejects_on_host(lib, over, code):
    assert _from_scores_call(lib, **over) == code


def test_select_from_scores_accepts_4_byte_rows_for_ragged_contexts(lib):
    # n_ctx not a multiple of 4: scores need only 4-byte alignment, so the
    # call passes every host check; it is not launched here (the workspace
    # is one byte short of its size, the last check)
    import lossless_ultra_long_b200 as L
    need = L.kv_select_from_scores_workspace_size(8, 2, 999)
    assert need > 0
    assert _from_scores_call(lib, rs=(1 << 20) + 4, n_ctx=999, ws_bytes=need - 1) == 3


def test_header_is_plain_c_and_the_library_serves_a_c_program(lib, tmp_path):
    """The public header compiles as C11 and as C++17, and a C program that
    loads libtsverify.so with dlopen finds every declared entry point and
    gets answers from the host-only ones (no device is touched)."""
    import subprocess
    from lossless_ultra_long_b200 import LIB_PATH
    inc = os.path.dirname(HEADER)
    names = declared_symbols()
    prog = tmp_path / "abi_c.c"
    prog.write_text(r"""
#include <dlfcn.h>
#include <stdio.h>
#include <string.h>
#include "ts_verify.h"
static const char *names[] = {%s};
int main(int argc, char **argv) {
    void *h = dlopen(argv[1], RTLD_NOW | RTLD_LOCAL);
    if (!h) { fprintf(stderr, "%%s\n", dlerror()); return 2; }
    for (size_t i = 0; i < sizeof names / sizeof names[0]; ++i)
        if (!dlsym(h, names[i])) { fprintf(stderr, "missing %%s\n", names[i]); return 3; }
    int (*version)(void) = (int (*)(void))dlsym(h, "ts_version");
    const char *(*status)(int) = (const char *(*)(int))dlsym(h, "ts_status_string");
    size_t (*ng_bytes)(int, int64_t) = (size_t (*)(int, int64_t))dlsym(h, "ts_ngram_table_bytes");
    int (*ng_init)(void *, size_t, int, int64_t) =
        (int (*)(void *, size_t, int, int64_t))dlsym(h, "ts_ngram_init");
    int (*ng_update)(void *, size_t, const int32_t *, int64_t, int64_t) =
        (int (*)(void *, size_t, const int32_t *, int64_t, int64_t))dlsym(h, "ts_ngram_update");
    int (*ng_topk)(const void *, size_t, int32_t, int, int32_t *, int64_t *, int *) =
        (int (*)(const void *, size_t, int32_t, int, int32_t *, int64_t *, int *))
            dlsym(h, "ts_ngram_topk");
    if (version() < 100 || strlen(status(TS_ERR_WORKSPACE)) == 0) return 4;
    static uint64_t table[(64 + 216 * 64) / 8];
    const size_t nb = ng_bytes(2, 64);
    if (nb != sizeof table || ng_init(table, nb, 2, 64) != TS_OK) return 5;
    const int32_t text[] = {5, 7, 5, 7, 5, 9};
    if (ng_update(table, nb, text, 6, 6) != TS_OK) return 6;
    int32_t cont[2]; int64_t cnt[2]; int found = 0;
    if (ng_topk(table, nb, 5, 2, cont, cnt, &found) != TS_OK) return 7;
    /* bigrams after 5: (5,7) twice, (5,9) once */
    if (found != 2 || cont[0] != 7 || cnt[0] != 2 || cont[1] != 9 || cnt[1] != 1) return 8;
    puts("ok");
    return 0;
}
""" % ", ".join('"%s"' % n for n in names))
    for lang, std in (("c", "-std=c11"), ("c++", "-std=c++17")):
        subprocess.run(["gcc", "-x", lang, std, "-fsyntax-only", "-Wall", "-Werror",
                        "-I", inc, "-"], input=b'#include "ts_verify.h"\n', check=True)
    exe = tmp_path / "abi_c"
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-I", inc, str(prog), "-o", str(exe),
                           "-ldl"])
    r = subprocess.run([str(exe), LIB_PATH], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stderr)
