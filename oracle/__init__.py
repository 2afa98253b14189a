"""CPU oracle for SparK channel pruning and recover-then-attend decode.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may import this module.
The product path never imports it and shares no code with it.

The arithmetic lives in ``spark_oracle.c`` (plain C, fp64, no fast-math); this
module only compiles it with gcc and marshals numpy arrays through ctypes.
Every function cites the passage of the SparK pages it follows; see the C
source header for the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spark_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, no FP contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        # ORACLE_LIB lets the planted-mistake tests run the pins against a
        # deliberately broken copy of the oracle.
        alt = os.environ.get("ORACLE_LIB")
        _lib = _bind(ctypes.CDLL(alt if alt else build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    L = ctypes.c_long
    I = ctypes.c_int
    lib.oracle_lambda_to_T.argtypes = [ctypes.c_float, I]
    lib.oracle_lambda_to_T.restype = I
    lib.oracle_qnorm.argtypes = [P, L, I, I, I, P]
    lib.oracle_qnorm.restype = None
    lib.oracle_prune.argtypes = [P, P, L, L, I, I, P, P, P]
    lib.oracle_prune.restype = None
    lib.oracle_recover_keys.argtypes = [P, P, P, P, L, L, I, I, P]
    lib.oracle_recover_keys.restype = None
    lib.oracle_decode.argtypes = [P, P, P, P, P, P, P, P, L, L, L, I, L, I, I, P]
    lib.oracle_decode.restype = None
    lib.oracle_philox4x32_10.argtypes = [P, P, P]
    lib.oracle_philox4x32_10.restype = None
    lib.oracle_sample_score.argtypes = [I, P, ctypes.c_ulonglong, L, L, I]
    lib.oracle_sample_score.restype = ctypes.c_double
    lib.oracle_recover_keys_f.argtypes = [P, P, P, P, L, L, I, I, I, ctypes.c_ulonglong, P]
    lib.oracle_recover_keys_f.restype = None
    lib.oracle_decode_f.argtypes = [P, P, P, P, P, P, P, P, L, L, L, I, L, I, I, I, ctypes.c_ulonglong, P]
    lib.oracle_decode_f.restype = None
    lib.oracle_snapkv_scores.argtypes = [P, P, L, I, I, L, I, P]
    lib.oracle_snapkv_scores.restype = None
    lib.oracle_snapkv_pool.argtypes = [P, L, L, I, P]
    lib.oracle_snapkv_pool.restype = None
    lib.oracle_snapkv_select.argtypes = [P, L, L, I, I, P]
    lib.oracle_snapkv_select.restype = None
    lib.oracle_group_of_channel.argtypes = [P, L, I, I, P]
    lib.oracle_group_of_channel.restype = None
    lib.oracle_group_budget.argtypes = [I, I, P, P]
    lib.oracle_group_budget.restype = None
    lib.oracle_pyramid_keep.argtypes = [I, I, ctypes.c_double, I, I, P]
    lib.oracle_pyramid_keep.restype = None
    lib.oracle_prune_grouped.argtypes = [P, P, L, L, I, I, P, P, P, P]
    lib.oracle_prune_grouped.restype = None
    lib.oracle_recover_values.argtypes = [P, P, L, L, I, I, P]
    lib.oracle_recover_values.restype = None
    lib.oracle_think_prune.argtypes = [P, P, L, L, I, I, P, P, P]
    lib.oracle_think_prune.restype = None
    lib.oracle_prune_topp.argtypes = [P, P, L, L, I, ctypes.c_float, I, P, P, P]
    lib.oracle_prune_topp.restype = None
    return lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def lambda_to_T(lam: float, D: int, lib=None) -> int:
    """T = round((1 - lambda) * D), half away from zero (reading R7)."""
    lib = lib or load()
    return int(lib.oracle_lambda_to_T(ctypes.c_float(lam), D))


def qnorm(q_obs, G: int, lib=None) -> np.ndarray:
    """Window-query channel norms.  q_obs: [BH*G, W, D] (or [B, Hq, W, D]).
    Returns qn [BH, D] fp32 (reading R1)."""
    lib = lib or load()
    q = _f32(q_obs)
    W, D = q.shape[-2], q.shape[-1]
    rows = q.size // (W * D)
    assert rows % G == 0
    BH = rows // G
    qn = np.empty((BH, D), np.float32)
    lib.oracle_qnorm(_ptr(q), BH, G, W, D, _ptr(qn))
    return qn


def prune(k, qn, T: int, lib=None):
    """Top-T channel pruning.  k: [BH, S, D]; qn: [BH, D].
    Returns (mask [BH, S, D/32] uint32, vals [BH, S, T] fp32,
    stats [BH, 4] fp64 = {N, sum w, sum w^2, mu})."""
    lib = lib or load()
    k = _f32(k)
    qn = _f32(qn)
    D = k.shape[-1]
    S = k.shape[-2]
    BH = k.size // (S * D) if S > 0 else qn.size // D
    nw = (D + 31) // 32
    mask = np.zeros((BH, S, nw), np.uint32)
    vals = np.zeros((BH, S, T), np.float32)
    stats = np.zeros((BH, 4), np.float64)
    lib.oracle_prune(_ptr(k), _ptr(qn), BH, S, D, T, _ptr(mask), _ptr(vals), _ptr(stats))
    return mask, vals, stats


def prune_topp(k, qn, p: float, Tcap: int, lib=None):
    """SparK-p pruning (reading R19): per token the shortest greedy prefix of
    channels whose fp32 saliency mass reaches fp32(p * total), at most Tcap
    channels.  k: [BH, S, D]; qn: [BH, D].  Returns (mask, vals [BH, S, Tcap]
    with the kept values first and zeros after, stats) in the layouts of
    prune()."""
    lib = lib or load()
    k = _f32(k)
    qn = _f32(qn)
    D = k.shape[-1]
    S = k.shape[-2]
    BH = int(np.prod(k.shape[:-2]))
    nw = (D + 31) // 32
    mask = np.zeros((BH, S, nw), np.uint32)
    vals = np.zeros((BH, S, Tcap), np.float32)
    stats = np.zeros((BH, 4), np.float64)
    lib.oracle_prune_topp(_ptr(k), _ptr(qn), BH, S, D, ctypes.c_float(p), Tcap, _ptr(mask), _ptr(vals),
                          _ptr(stats))
    return mask, vals, stats


def group_of_channel(qn, g: int, lib=None) -> np.ndarray:
    """SparK-g channel groups by window-query norm rank (reading R15).
    qn: [BH, D] -> gid [BH, D] int32."""
    lib = lib or load()
    qn = _f32(qn)
    D = qn.shape[-1]
    BH = qn.size // D
    gid = np.zeros((BH, D), np.int32)
    lib.oracle_group_of_channel(_ptr(qn), BH, D, g, _ptr(gid))
    return gid


def pyramid_keep(L: int, M: int, beta: float, W: int, S: int, lib=None) -> list:
    """PyramidKV-style layer budgets (reading R20); beta is taken as the
    fp32 value the C library receives."""
    lib = lib or load()
    out = np.zeros(max(L, 1), np.int32)
    lib.oracle_pyramid_keep(L, M, float(np.float32(beta)), W, S, _ptr(out))
    return [int(x) for x in out[:L]]


def group_budget(D: int, rates, lib=None) -> list:
    """Per-group kept-channel budgets from pruning rates (reading R15)."""
    lib = lib or load()
    r = _f32(rates)
    Tg = np.zeros(len(r), np.int32)
    lib.oracle_group_budget(D, len(r), _ptr(r), _ptr(Tg))
    return [int(x) for x in Tg]


def prune_grouped(k, qn, Tg, lib=None):
    """SparK-g pruning (reading R15).  k: [BH, S, D]; qn: [BH, D]; Tg: one
    kept-channel budget per group.  Returns (mask, vals [BH, S, sum Tg],
    stats) in the layouts of prune()."""
    lib = lib or load()
    k = _f32(k)
    qn = _f32(qn)
    D = k.shape[-1]
    S = k.shape[-2]
    BH = k.size // (S * D) if S > 0 else qn.size // D
    tg = np.ascontiguousarray(Tg, np.int32)
    T = int(tg.sum())
    nw = (D + 31) // 32
    mask = np.zeros((BH, S, nw), np.uint32)
    vals = np.zeros((BH, S, T), np.float32)
    stats = np.zeros((BH, 4), np.float64)
    lib.oracle_prune_grouped(_ptr(k), _ptr(qn), BH, S, D, len(tg), _ptr(tg), _ptr(mask), _ptr(vals),
                             _ptr(stats))
    return mask, vals, stats


def think_prune(k, qn, T: int, lib=None):
    """ThinK structured pruning (reading R18): one channel mask per (b, h),
    channels ranked by qn_j * ||k^j||_2 over the tokens.  Returns (mask, vals,
    stats) in the layouts of prune(); stats = {N, 0, 0, 0} (no recovery)."""
    lib = lib or load()
    k = _f32(k)
    qn = _f32(qn)
    D = k.shape[-1]
    S = k.shape[-2]
    BH = int(np.prod(k.shape[:-2]))
    nw = (D + 31) // 32
    mask = np.zeros((BH, S, nw), np.uint32)
    vals = np.zeros((BH, S, T), np.float32)
    stats = np.zeros((BH, 4), np.float64)
    lib.oracle_think_prune(_ptr(k), _ptr(qn), BH, S, D, T, _ptr(mask), _ptr(vals), _ptr(stats))
    return mask, vals, stats


def prune_values(v, Tv: int, lib=None):
    """V-channel pruning (reading R16): top-T_v channels of |v| per token,
    i.e. prune() with unit query norms.  v: [BH, S, D].  Returns
    (vmask, vvals, stats) in the layouts of prune()."""
    v = _f32(v)
    D = v.shape[-1]
    BH = int(np.prod(v.shape[:-2]))
    return prune(v.reshape(BH, v.shape[-2], D), np.ones((BH, D), np.float32), Tv, lib=lib)


def recover_values(vmask, vvals, bh: int, lib=None) -> np.ndarray:
    """Dense recovered value block V^ [S, D] (fp64) of one (b, h): kept
    values, 0 on pruned channels (reading R16)."""
    lib = lib or load()
    vmask = np.ascontiguousarray(vmask, np.uint32)
    vvals = _f32(vvals)
    S = vmask.shape[-2]
    D = vmask.shape[-1] * 32
    Tv = vvals.shape[-1]
    out = np.zeros((S, D), np.float64)
    lib.oracle_recover_values(_ptr(vmask), _ptr(vvals), bh, S, D, Tv, _ptr(out))
    return out


def decode_kv(q, mask, vals, qn, stats, vmask, vvals, k_tail=None, v_tail=None, n_tail: int = 0, G: int = 1,
              lib=None) -> np.ndarray:
    """Decode over a pruned key cache and a pruned value cache: the value
    rows are the recovered V^ of recover_values (R16), then decode()."""
    vmask = np.ascontiguousarray(vmask, np.uint32)
    BH, S = vmask.shape[0], vmask.shape[1]
    D = vmask.shape[-1] * 32
    vhat = np.zeros((BH, S, D), np.float32)
    for bh in range(BH):
        vhat[bh] = recover_values(vmask, vvals, bh, lib=lib).astype(np.float32)  # exact: kept values are fp32
    return decode(q, mask, vals, qn, stats, vhat, k_tail, v_tail, n_tail, G, lib=lib)


def recover_keys(mask, vals, qn, stats, bh: int, lib=None) -> np.ndarray:
    """Dense recovered key block K~ [S, D] (fp64) of one (b, h)."""
    lib = lib or load()
    mask = np.ascontiguousarray(mask, np.uint32)
    vals = _f32(vals)
    qn = _f32(qn)
    stats = np.ascontiguousarray(stats, np.float64)
    BH, S, _ = mask.shape
    D = qn.shape[-1]
    T = vals.shape[-1]
    out = np.empty((S, D), np.float64)
    lib.oracle_recover_keys(_ptr(mask), _ptr(vals), _ptr(qn), _ptr(stats), bh, S, D, T, _ptr(out))
    return out


def decode(q, mask, vals, qn, stats, v, k_tail=None, v_tail=None, n_tail: int = 0,
           G: int = 1, lib=None) -> np.ndarray:
    """Recover-then-attend decode.  q: [BH*G, D]; v: [BH, S, D];
    k_tail/v_tail: [BH, cap, D].  Returns out [BH*G, D] fp32."""
    lib = lib or load()
    q = _f32(q)
    mask = np.ascontiguousarray(mask, np.uint32)
    vals = _f32(vals)
    qn = _f32(qn)
    stats = np.ascontiguousarray(stats, np.float64)
    v = _f32(v)
    BH, D = qn.shape
    S = mask.shape[1]
    T = vals.shape[-1]
    if k_tail is None:
        cap = max(n_tail, 1)
        k_tail = np.zeros((BH, cap, D), np.float32)
        v_tail = np.zeros((BH, cap, D), np.float32)
    k_tail = _f32(k_tail)
    v_tail = _f32(v_tail)
    cap = k_tail.shape[1]
    assert 0 <= n_tail <= cap
    out = np.empty((BH * G, D), np.float32)
    lib.oracle_decode(_ptr(q), _ptr(mask), _ptr(vals), _ptr(qn), _ptr(stats), _ptr(v),
                      _ptr(k_tail), _ptr(v_tail), cap, n_tail, BH, G, S, D, T, _ptr(out))
    return out


def snapkv_scores(q_obs, k, G: int, lib=None) -> np.ndarray:
    """Summed window-attention probabilities of the prefix tokens (reading
    R11).  q_obs: [BH*G, W, D]; k: [BH, S, D].  Returns [BH, S-W] fp64."""
    lib = lib or load()
    q = _f32(q_obs)
    k = _f32(k)
    BH, S, D = k.shape
    W = q.shape[-2]
    out = np.zeros((BH, max(S - W, 0)), np.float64)
    lib.oracle_snapkv_scores(_ptr(q), _ptr(k), BH, G, W, S, D, _ptr(out))
    return out


def snapkv_pool(scores, pool: int, lib=None) -> np.ndarray:
    """1-D max-pool of the scores along tokens (reading R12)."""
    lib = lib or load()
    sc = np.ascontiguousarray(scores, np.float64)
    BH, P = sc.shape
    out = np.empty_like(sc)
    lib.oracle_snapkv_pool(_ptr(sc), BH, P, pool, _ptr(out))
    return out


def snapkv_select(pooled, S: int, W: int, keep: int, lib=None) -> np.ndarray:
    """Kept token indices [BH, keep] in original order (reading R13)."""
    lib = lib or load()
    pl = np.ascontiguousarray(pooled, np.float64)
    BH = pl.shape[0]
    idx = np.empty((BH, keep), np.int64)
    lib.oracle_snapkv_select(_ptr(pl), BH, S, W, keep, _ptr(idx))
    return idx


DEGENERATE, GAUSSIAN, EXPONENTIAL = 0, 1, 2


def philox4x32_10(ctr, key, lib=None):
    """Philox4x32-10 of one counter block (reading R14)."""
    lib = lib or load()
    c = np.ascontiguousarray(ctr, np.uint32)
    k = np.ascontiguousarray(key, np.uint32)
    out = np.empty(4, np.uint32)
    lib.oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sample_score(mode: int, stats_row, seed: int, bh: int, t: int, j: int, lib=None) -> float:
    lib = lib or load()
    st = np.ascontiguousarray(stats_row, np.float64)
    return float(lib.oracle_sample_score(mode, _ptr(st), seed, bh, t, j))


def recover_keys_f(mask, vals, qn, stats, bh: int, mode: int, seed: int, lib=None) -> np.ndarray:
    lib = lib or load()
    mask = np.ascontiguousarray(mask, np.uint32)
    vals = _f32(vals)
    qn = _f32(qn)
    stats = np.ascontiguousarray(stats, np.float64)
    BH, S, _ = mask.shape
    D = qn.shape[-1]
    T = vals.shape[-1]
    out = np.empty((S, D), np.float64)
    lib.oracle_recover_keys_f(_ptr(mask), _ptr(vals), _ptr(qn), _ptr(stats), bh, S, D, T, mode, seed, _ptr(out))
    return out


def decode_f(q, mask, vals, qn, stats, v, k_tail=None, v_tail=None, n_tail: int = 0, G: int = 1,
             mode: int = DEGENERATE, seed: int = 0, lib=None) -> np.ndarray:
    """Decode with recovery F (Degenerate, Gaussian or Exponential)."""
    lib = lib or load()
    q = _f32(q)
    mask = np.ascontiguousarray(mask, np.uint32)
    vals = _f32(vals)
    qn = _f32(qn)
    stats = np.ascontiguousarray(stats, np.float64)
    v = _f32(v)
    BH, D = qn.shape
    S = mask.shape[1]
    T = vals.shape[-1]
    if k_tail is None:
        cap = max(n_tail, 1)
        k_tail = np.zeros((BH, cap, D), np.float32)
        v_tail = np.zeros((BH, cap, D), np.float32)
    k_tail = _f32(k_tail)
    v_tail = _f32(v_tail)
    cap = k_tail.shape[1]
    out = np.empty((BH * G, D), np.float32)
    lib.oracle_decode_f(_ptr(q), _ptr(mask), _ptr(vals), _ptr(qn), _ptr(stats), _ptr(v), _ptr(k_tail),
                        _ptr(v_tail), cap, n_tail, BH, G, S, D, T, mode, seed, _ptr(out))
    return out
