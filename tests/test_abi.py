"""Host-side checks of the C ABI library (no GPU needed): it builds and
loads, exports exactly what include/spark.h declares, and its host logic
(lambda -> T, cache layout sizes, workspace sizes, argument validation)
behaves as documented.  No compute call is made."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from channel_pruned_decode_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spark.h")


@pytest.fixture(scope="module")
def L():
    from channel_pruned_decode_b200 import build
    build.build()
    return B.lib()


def _declared():
    txt = open(HEADER).read()
    return set(re.findall(r"SPARK_API\s+[\w\s\*]*?\b(spark_\w+)\s*\(", txt))


def test_exports_match_header(L):
    decl = _declared()
    assert decl == set(B.EXPORTS)
    for name in decl:
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", B._LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln and "spark" in ln}
    assert exported == decl


@pytest.mark.parametrize("lam", [0.0, 0.1, 0.25, 0.3, 0.5, 0.58, 0.8, 0.9, 1.0, -0.01, 1.01])
def test_lambda_to_T_matches_oracle(L, lam):
    assert B.spark_lambda_to_T(lam, 128) == oracle.lambda_to_T(lam, 128)


def test_cache_sizes_layout():
    for (b, h, s, t, dt, es) in [(1, 8, 32768, 64, B.SPARK_BF16, 2), (2, 2, 513, 26, B.SPARK_F32, 4),
                                 (1, 1, 0, 0, B.SPARK_BF16, 2)]:
        total, sz = B.spark_cache_sizes(b, h, s, 128, t, dt)
        s32 = (s + 31) // 32 * 32
        assert sz == [b * h * s * 16, b * h * s32 * t * es, b * h * 128 * 4, b * h * 32]
        assert total == sum((x + 255) // 256 * 256 for x in sz)
        assert B.spark_cache_bytes(b, h, s, 128, t, dt) == total
    assert B.spark_cache_bytes(1, 1, 16, 64, 8, B.SPARK_BF16) == 0       # D != 128
    assert B.spark_cache_bytes(1, 1, 16, 128, 129, B.SPARK_BF16) == 0    # T > D
    assert B.spark_cache_bytes(1, 1, 16, 128, 8, 7) == 0                 # dtype


def test_storage_reduction_arithmetic():
    # key bytes per token-head: 16-byte mask + T kept bf16 values vs 256 dense.
    # lambda 0.5 -> 144 B (43.75 % smaller key, 21.9 % smaller K+V);
    # lambda 0.8 -> 68 B (73.4 % smaller key, 36.7 % smaller K+V) -- the pages
    # quote ~50 % key / ~25 % total and ~40 % total without the mask overhead.
    S = 1 << 15
    for lam, key_red, kv_red in [(0.5, 0.4375, 0.21875), (0.8, 0.734375, 0.3671875)]:
        T = B.spark_lambda_to_T(lam, 128)
        _, sz = B.spark_cache_sizes(1, 1, S, 128, T, B.SPARK_BF16)
        per_tok = (sz[0] + sz[1]) / S
        assert 1 - per_tok / 256 == pytest.approx(key_red)
        assert 1 - (per_tok + 256) / 512 == pytest.approx(kv_red)


def test_workspace_sizes():
    assert B.spark_workspace_bytes(B.SPARK_OP_PRUNE, 1, 8, 4, 32768, 128, 64, 0) >= 256 + 8 * 128 * 16
    assert B.spark_workspace_bytes(B.SPARK_OP_DECODE, 1, 8, 4, 32768, 128, 64, 256) > 256
    assert B.spark_workspace_bytes(B.SPARK_OP_DECODE, 1, 8, 3, 32768, 128, 64, 256) == 0  # G
    assert B.spark_workspace_bytes(B.SPARK_OP_PRUNE, 1, 8, 4, 32768, 96, 64, 0) == 0      # D
    assert B.spark_workspace_bytes(9, 1, 8, 4, 32768, 128, 64, 0) == 0                   # op


def _kc(**kw):
    d = dict(B=1, Hkv=2, S=64, D=128, T=32, dtype=B.SPARK_BF16, mask=16, vals=16, qn=16, stats=16)
    d.update(kw)
    return B.spark_kcache(**d)


@pytest.mark.parametrize("kw,want", [
    (dict(D=64), B.SPARK_ERR_UNSUPPORTED),
    (dict(T=129), B.SPARK_ERR_ARG),
    (dict(T=-1), B.SPARK_ERR_ARG),
    (dict(dtype=5), B.SPARK_ERR_ARG),
    (dict(mask=None), B.SPARK_ERR_ARG),
    (dict(vals=24), B.SPARK_ERR_ARG),   # misaligned
    (dict(S=-1), B.SPARK_ERR_ARG),
])
def test_prune_rejects_bad_cache(L, kw, want):
    kc = _kc(**kw)
    rc = L.spark_prune(16, 16, 4, 32, ctypes.byref(kc), 256, 1 << 20, None)
    assert rc == want


def test_prune_rejects_bad_args(L):
    kc = _kc()
    assert L.spark_prune(16, 16, 0, 32, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert L.spark_prune(16, 16, 4, 0, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert L.spark_prune(None, 16, 4, 32, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert L.spark_prune(16, 16, 4, 32, ctypes.byref(kc), None, 1 << 20, None) == B.SPARK_ERR_WORKSPACE
    assert L.spark_prune(16, 16, 4, 32, ctypes.byref(kc), 256, 16, None) == B.SPARK_ERR_WORKSPACE
    assert L.spark_prune(16, 16, 4, 32, None, 256, 1 << 20, None) == B.SPARK_ERR_ARG


def test_decode_rejects_bad_args(L):
    kc = _kc()
    call = lambda **k: L.spark_decode_attn(
        k.get("q", 16), ctypes.byref(kc), k.get("v", 16), k.get("kt", 16), k.get("vt", 16),
        k.get("cap", 8), k.get("n", 0), k.get("G", 4), k.get("rec", 0), 0, k.get("out", 16),
        k.get("ws", 256), 1 << 20, None)
    assert call(G=3) == B.SPARK_ERR_UNSUPPORTED
    assert call(G=0) == B.SPARK_ERR_ARG
    # (every call here must fail validation: the pointers are not real)
    assert call(rec=B.SPARK_F_GAUSSIAN, ws=None) == B.SPARK_ERR_WORKSPACE
    assert call(rec=B.SPARK_F_EXPONENTIAL, G=3) == B.SPARK_ERR_UNSUPPORTED
    assert call(rec=9) == B.SPARK_ERR_ARG
    assert call(n=9) == B.SPARK_ERR_ARG          # n_tail > tail_cap
    assert call(cap=-1) == B.SPARK_ERR_ARG
    assert call(q=None) == B.SPARK_ERR_ARG
    assert call(out=8) == B.SPARK_ERR_ARG        # misaligned
    assert call(kt=None) == B.SPARK_ERR_ARG      # tail_cap > 0 needs tail buffers
    assert call(ws=None) == B.SPARK_ERR_WORKSPACE


def test_tail_append_rejects_bad_args(L):
    f = L.spark_tail_append
    assert f(16, 16, 16, 16, 1, 2, 64, 8, 0, B.SPARK_BF16, None) == B.SPARK_ERR_UNSUPPORTED
    assert f(16, 16, 16, 16, 1, 2, 128, 8, 8, B.SPARK_BF16, None) == B.SPARK_ERR_ARG   # slot
    assert f(16, 16, 16, 16, 1, 2, 128, 0, 0, B.SPARK_BF16, None) == B.SPARK_ERR_ARG   # cap
    assert f(None, 16, 16, 16, 1, 2, 128, 8, 0, B.SPARK_BF16, None) == B.SPARK_ERR_ARG
    assert f(16, 16, 16, 16, 1, 2, 128, 8, 0, 3, None) == B.SPARK_ERR_ARG


def test_status_strings(L):
    for s in range(6):
        assert B.status_str(s)
    assert B.status_str(99) == "unknown status"


def test_empty_batch_is_a_no_op(L):
    kc = _kc(B=0)
    assert L.spark_prune(None, None, 4, 32, ctypes.byref(kc), None, 0, None) == B.SPARK_OK


def test_snapkv_rejects_bad_args(L):
    f = lambda **k: L.spark_snapkv_evict(16, 16, 16, 1, 2, k.get("S", 256), k.get("D", 128), k.get("G", 4),
                                         k.get("W", 32), k.get("keep", 64), k.get("pool", 7),
                                         k.get("dt", B.SPARK_BF16), 16, 16, 16, k.get("ws", None), 1 << 20, None)
    assert f(D=64) == B.SPARK_ERR_UNSUPPORTED
    assert f(dt=B.SPARK_F32) == B.SPARK_ERR_UNSUPPORTED
    assert f(G=3, W=5) == B.SPARK_ERR_UNSUPPORTED     # G*W not a multiple of 16
    assert f(G=8, W=32) == B.SPARK_ERR_UNSUPPORTED    # G*W > 128
    assert f(keep=16) == B.SPARK_ERR_ARG              # keep < W
    assert f(keep=300) == B.SPARK_ERR_ARG             # keep > S
    assert f(pool=6) == B.SPARK_ERR_ARG               # even pool
    assert f() == B.SPARK_ERR_WORKSPACE               # no workspace


def test_prune_grouped_rejects_bad_budgets(L):
    # every call here must fail validation: the pointers are not real
    kc = _kc()  # T = 32
    I = ctypes.c_int
    f = lambda tg, n=None, **k: L.spark_prune_grouped(
        16, 16, k.get("G", 4), 32, len(tg) if n is None else n, (I * max(len(tg), 1))(*tg),
        ctypes.byref(kc), k.get("ws", 256), 1 << 20, None)
    assert f([10, 10, 5]) == B.SPARK_ERR_ARG             # sum 25 != T
    assert f([33, 0, -1]) == B.SPARK_ERR_ARG             # negative budget
    assert f([26, 0]) == B.SPARK_ERR_ARG                 # sum 26 != T
    assert f([32], n=0) == B.SPARK_ERR_ARG               # no groups
    assert f([4] * 8 + [0]) == B.SPARK_ERR_ARG           # more than 8 groups
    assert f([16, 16], G=0) == B.SPARK_ERR_ARG
    assert f([0] * 7 + [32]) == B.SPARK_ERR_ARG          # 32 > group size 16
    assert L.spark_prune_grouped(16, 16, 4, 32, 2, None, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert f([16, 16], ws=None) == B.SPARK_ERR_WORKSPACE


def test_group_budget_matches_oracle():
    for rates in ([0.25, 0.5, 0.75, 1.0], [0.5] * 5, [0.1, 0.3, 0.5, 0.7, 0.9], [0.0] * 8, [1.0] * 3, [0.33] * 7):
        assert B.spark_group_budget(128, rates) == oracle.group_budget(128, rates)
    # the pages' g = 4 rates over 128 channels: groups of 32 keep 24, 16, 8, 0
    assert B.spark_group_budget(128, [0.25, 0.5, 0.75, 1.0]) == [24, 16, 8, 0]


def test_group_budget_rejects_bad_args(L):
    F, I = ctypes.c_float, ctypes.c_int
    rates, out = (F * 9)(*([0.5] * 9)), (I * 9)(*([-7] * 9))
    assert L.spark_group_budget(128, 0, rates, out) == B.SPARK_ERR_ARG        # no groups
    assert L.spark_group_budget(128, 9, rates, out) == B.SPARK_ERR_ARG        # more than 8
    assert L.spark_group_budget(2, 4, rates, out) == B.SPARK_ERR_ARG          # more groups than channels
    assert L.spark_group_budget(0, 1, rates, out) == B.SPARK_ERR_ARG
    assert L.spark_group_budget(128, 4, None, out) == B.SPARK_ERR_ARG
    assert L.spark_group_budget(128, 4, rates, None) == B.SPARK_ERR_ARG
    for bad in (-0.01, 1.01, float("nan")):
        r = (F * 4)(0.5, bad, 0.5, 0.5)
        assert L.spark_group_budget(128, 4, r, out) == B.SPARK_ERR_ARG
    assert list(out) == [-7] * 9                                             # untouched on error


C_PROGRAM = r"""
#include <math.h>
#include <stdio.h>
#include "spark.h"

int main(void) {
    /* lambda -> T and the cache / workspace sizes are host arithmetic */
    if (spark_lambda_to_T(0.8f, 128) != 26 || spark_lambda_to_T(1.5f, 128) != -1) return 1;
    size_t sizes[4];
    const size_t total = spark_cache_sizes(1, 8, 32768, 128, 64, SPARK_BF16, sizes);
    if (total == 0 || sizes[0] != (size_t)8 * 32768 * 16) return 2;
    if (spark_cache_bytes(1, 8, 32768, 128, 64, SPARK_BF16) != total) return 3;
    if (spark_workspace_bytes(SPARK_OP_PRUNE, 1, 8, 4, 32768, 128, 64, 0) == 0) return 4;
    if (spark_workspace_bytes(SPARK_OP_PRUNE, 1, 8, 4, 32768, 64, 64, 0) != 0) return 5;
    const float rates[4] = {0.25f, 0.5f, 0.75f, 1.0f};
    int Tg[4];
    if (spark_group_budget(128, 4, rates, Tg) != SPARK_OK) return 6;
    if (Tg[0] != 24 || Tg[1] != 16 || Tg[2] != 8 || Tg[3] != 0) return 7;
    /* argument errors come back before anything is launched */
    if (spark_prune(NULL, NULL, 4, 32, NULL, NULL, 0, NULL) != SPARK_ERR_ARG) return 8;
    spark_kcache kc = {0};
    kc.B = 1; kc.Hkv = 8; kc.S = 32768; kc.D = 96; kc.T = 64; kc.dtype = SPARK_BF16;
    if (spark_prune(NULL, NULL, 4, 32, &kc, NULL, 0, NULL) != SPARK_ERR_UNSUPPORTED) return 9;
    if (spark_status_str(SPARK_ERR_ARG) == NULL) return 10;
    printf("ok %zu\n", total);
    return 0;
}
"""


def test_header_compiles_as_c_and_links(L, tmp_path):
    # a C11 caller: the header must be valid C on its own, and the calls above
    # must link against and run with libspark.so (host arithmetic and argument
    # errors only, so no GPU is needed)
    src = tmp_path / "caller.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(B._LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lspark",
                    f"-Wl,-rpath,{libdir}", "-lm"], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok ")


def test_value_pruning_entry_points_reject_bad_args(L):
    # every call here must fail validation: the pointers are not real
    kc, vc = _kc(), _kc(T=64)
    f = lambda k=kc, v=vc, **a: L.spark_decode_attn_kv(
        a.get("q", 16), ctypes.byref(k), ctypes.byref(v), 16, 16, a.get("cap", 8), a.get("n", 0), a.get("G", 4),
        a.get("out", 16), a.get("ws", 256), 1 << 20, None)
    assert f(v=_kc(T=64, S=32)) == B.SPARK_ERR_ARG                      # shapes differ
    assert f(k=_kc(dtype=B.SPARK_F32), v=_kc(T=64, dtype=B.SPARK_F32)) == B.SPARK_ERR_UNSUPPORTED
    assert f(G=3) == B.SPARK_ERR_UNSUPPORTED
    assert f(n=9) == B.SPARK_ERR_ARG
    assert f(q=None) == B.SPARK_ERR_ARG
    assert f(ws=None) == B.SPARK_ERR_WORKSPACE
    assert L.spark_workspace_bytes_kv(1, 2, 4, 64, 128, 26, 129, 8) == 0
    assert L.spark_workspace_bytes_kv(1, 2, 3, 64, 128, 26, 64, 8) == 0
    assert L.spark_prune_values(16, ctypes.byref(_kc(T=129)), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert L.spark_prune_values(None, ctypes.byref(vc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert L.spark_prune_values(16, ctypes.byref(vc), None, 1 << 20, None) == B.SPARK_ERR_WORKSPACE


def test_prune_think_rejects_bad_args(L):
    kc = _kc()
    f = L.spark_prune_think
    assert f(16, 16, 0, 32, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert f(16, 16, 4, 0, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert f(None, 16, 4, 32, ctypes.byref(kc), 256, 1 << 20, None) == B.SPARK_ERR_ARG
    assert f(16, 16, 4, 32, ctypes.byref(kc), None, 1 << 20, None) == B.SPARK_ERR_WORKSPACE
    assert f(16, 16, 4, 32, ctypes.byref(kc), 256, 64, None) == B.SPARK_ERR_WORKSPACE
    assert f(16, 16, 4, 32, ctypes.byref(_kc(T=129)), 256, 1 << 20, None) == B.SPARK_ERR_ARG


def test_prune_topp_rejects_bad_args(L):
    kc = _kc(goff=16)

    def f(p=0.99, k=16, G=4, c=None, ws=256, wsb=1 << 20):
        return L.spark_prune_topp(k, 16, G, 32, ctypes.c_float(p), ctypes.byref(c or kc), ws, wsb, None)
    for p in (1.5, -0.1, float("nan")):
        assert f(p=p) == B.SPARK_ERR_ARG
    assert f(G=0) == B.SPARK_ERR_ARG
    assert f(k=None) == B.SPARK_ERR_ARG
    assert f(ws=None) == B.SPARK_ERR_WORKSPACE
    assert f(wsb=64) == B.SPARK_ERR_WORKSPACE
    assert f(c=_kc(T=129, goff=16)) == B.SPARK_ERR_ARG
    assert f(c=_kc(D=64, goff=16)) == B.SPARK_ERR_UNSUPPORTED
    assert f(c=_kc()) == B.SPARK_ERR_ARG                     # no group offsets
    assert f(c=_kc(goff=18)) == B.SPARK_ERR_ARG              # misaligned offsets
    # value rows counted in 32 bits: 2^20 heads x 2^11 groups x 128 slots is too many
    assert f(c=_kc(B=1 << 10, Hkv=1 << 10, S=1 << 16, T=128, goff=16)) == B.SPARK_ERR_UNSUPPORTED
    # three fp64 partials per chunk of 256 tokens (the pruned count is the third)
    assert B.spark_workspace_bytes(B.SPARK_OP_TOPP, 1, 8, 4, 32768, 128, 128, 0) >= 256 + 8 * 128 * 24
    assert B.spark_workspace_bytes(B.SPARK_OP_TOPP, 1, 8, 4, 32768, 128, 128, 0) > \
        B.spark_workspace_bytes(B.SPARK_OP_PRUNE, 1, 8, 4, 32768, 128, 128, 0)


def test_topp_offsets_bytes(L):
    assert B.spark_topp_offsets_bytes(1, 8, 32768) == (8 * 1024 + 1) * 4
    assert B.spark_topp_offsets_bytes(2, 3, 33) == (2 * 3 * 2 + 1) * 4
    assert B.spark_topp_offsets_bytes(1, 1, 0) == 4
    assert B.spark_topp_offsets_bytes(-1, 1, 5) == 0
    n = ctypes.c_size_t(7)
    assert L.spark_topp_vals_used(ctypes.byref(_kc()), ctypes.byref(n), None) == B.SPARK_ERR_ARG  # no goff
    assert L.spark_topp_vals_used(None, ctypes.byref(n), None) == B.SPARK_ERR_ARG
    assert n.value == 7


def test_decode_topp_rejects_bad_args(L):
    kc = _kc(goff=16)
    call = lambda **k: L.spark_decode_attn_topp(
        k.get("q", 16), ctypes.byref(kc), k.get("v", 16), k.get("kt", 16), k.get("vt", 16),
        k.get("cap", 8), k.get("n", 0), k.get("G", 4), k.get("rec", 0), 0, k.get("out", 16),
        k.get("ws", 256), 1 << 20, None)
    assert call(G=3) == B.SPARK_ERR_UNSUPPORTED
    assert call(rec=9) == B.SPARK_ERR_ARG
    assert call(n=9) == B.SPARK_ERR_ARG
    assert call(q=None) == B.SPARK_ERR_ARG
    assert call(kt=None) == B.SPARK_ERR_ARG
    assert call(ws=None) == B.SPARK_ERR_WORKSPACE
    kc.goff = None
    assert call() == B.SPARK_ERR_ARG  # a SparK-p decode needs the group offsets
