"""Thin ctypes binding of libspark.so (include/spark.h).

Argument marshalling only: every step of pruning and decode runs in the CUDA
kernels of libspark.so.  torch tensors supply device memory and streams.
There is no CPU fallback: loading fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspark.so")

SPARK_OK = 0
SPARK_ERR_ARG = 1
SPARK_ERR_UNSUPPORTED = 2
SPARK_ERR_CUDA = 3
SPARK_ERR_TIMEOUT = 4
SPARK_ERR_WORKSPACE = 5
SPARK_F32 = 0
SPARK_BF16 = 1
SPARK_F_DEGENERATE = 0
SPARK_F_GAUSSIAN = 1
SPARK_F_EXPONENTIAL = 2
SPARK_OP_PRUNE = 0
SPARK_OP_DECODE = 1
SPARK_OP_SNAPKV = 2
SPARK_OP_THINK = 3
SPARK_OP_TOPP = 4

EXPORTS = ("spark_lambda_to_T", "spark_cache_sizes", "spark_cache_bytes", "spark_workspace_bytes",
           "spark_prune", "spark_prune_noalloc", "spark_prune_grouped", "spark_group_budget", "spark_prune_values", "spark_prune_think", "spark_prune_topp", "spark_decode_attn",
           "spark_decode_attn_topp", "spark_topp_offsets_bytes", "spark_topp_vals_used",
           "spark_decode_attn_kv", "spark_workspace_bytes_kv", "spark_selftest_wait_timeout", "spark_tail_append", "spark_device_status",
           "spark_status_str", "spark_snapkv_evict", "spark_snapkv_evict_rows", "spark_pyramid_keep")


class SparkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


class spark_kcache(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("S", ctypes.c_int), ("D", ctypes.c_int),
                ("T", ctypes.c_int), ("dtype", ctypes.c_int), ("mask", ctypes.c_void_p),
                ("vals", ctypes.c_void_p), ("qn", ctypes.c_void_p), ("stats", ctypes.c_void_p),
                ("goff", ctypes.c_void_p), ("lens", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libspark.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"SparK CUDA library not found at {_LIB_PATH}; build it with "
                               "`python -m channel_pruned_decode_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.spark_lambda_to_T.argtypes = [ctypes.c_float, I]
        L.spark_lambda_to_T.restype = I
        L.spark_cache_sizes.argtypes = [I, I, I, I, I, I, ctypes.POINTER(Z)]
        L.spark_cache_sizes.restype = Z
        L.spark_cache_bytes.argtypes = [I, I, I, I, I, I]
        L.spark_cache_bytes.restype = Z
        L.spark_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I]
        L.spark_workspace_bytes.restype = Z
        L.spark_prune.argtypes = [P, P, I, I, ctypes.POINTER(spark_kcache), P, Z, P]
        L.spark_prune.restype = I
        L.spark_prune_noalloc.argtypes = [P, P, I, I, ctypes.POINTER(spark_kcache), P]
        L.spark_prune_noalloc.restype = I
        L.spark_prune_grouped.argtypes = [P, P, I, I, I, ctypes.POINTER(I), ctypes.POINTER(spark_kcache), P, Z, P]
        L.spark_prune_grouped.restype = I
        L.spark_group_budget.argtypes = [I, I, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(I)]
        L.spark_group_budget.restype = I
        L.spark_prune_values.argtypes = [P, ctypes.POINTER(spark_kcache), P, Z, P]
        L.spark_prune_values.restype = I
        L.spark_prune_think.argtypes = [P, P, I, I, ctypes.POINTER(spark_kcache), P, Z, P]
        L.spark_prune_think.restype = I
        L.spark_prune_topp.argtypes = [P, P, I, I, ctypes.c_float, ctypes.POINTER(spark_kcache), P, Z, P]
        L.spark_prune_topp.restype = I
        L.spark_decode_attn_topp.argtypes = [P, ctypes.POINTER(spark_kcache), P, P, P, I, I, I, I,
                                             ctypes.c_ulonglong, P, P, Z, P]
        L.spark_decode_attn_topp.restype = I
        L.spark_topp_offsets_bytes.argtypes = [I, I, I]
        L.spark_topp_offsets_bytes.restype = Z
        L.spark_topp_vals_used.argtypes = [ctypes.POINTER(spark_kcache), ctypes.POINTER(Z), P]
        L.spark_topp_vals_used.restype = I
        L.spark_selftest_wait_timeout.argtypes = [P, I, P]
        L.spark_selftest_wait_timeout.restype = I
        L.spark_decode_attn_kv.argtypes = [P, ctypes.POINTER(spark_kcache), ctypes.POINTER(spark_kcache), P, P, I,
                                           I, I, P, P, Z, P]
        L.spark_decode_attn_kv.restype = I
        L.spark_workspace_bytes_kv.argtypes = [I, I, I, I, I, I, I, I]
        L.spark_workspace_bytes_kv.restype = Z
        L.spark_decode_attn.argtypes = [P, ctypes.POINTER(spark_kcache), P, P, P, I, I, I, I,
                                        ctypes.c_ulonglong, P, P, Z, P]
        L.spark_decode_attn.restype = I
        L.spark_snapkv_evict.argtypes = [P, P, P, I, I, I, I, I, I, I, I, I, P, P, P, P, Z, P]
        L.spark_snapkv_evict.restype = I
        L.spark_snapkv_evict_rows.argtypes = [P, P, P, I, I, I, I, I, I, P, I, I, I, P, P, P, P, Z, P]
        L.spark_snapkv_evict_rows.restype = I
        L.spark_pyramid_keep.argtypes = [I, I, ctypes.c_float, I, I, ctypes.POINTER(I)]
        L.spark_pyramid_keep.restype = I
        L.spark_tail_append.argtypes = [P, P, P, P, I, I, I, I, I, I, P]
        L.spark_tail_append.restype = I
        L.spark_device_status.argtypes = [P, ctypes.POINTER(I), I, P]
        L.spark_device_status.restype = I
        L.spark_status_str.argtypes = [I]
        L.spark_status_str.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().spark_status_str(status).decode()


def _check(rc: int, where: str):
    if rc != SPARK_OK:
        raise SparkError(rc, where)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return SPARK_BF16
    if t == torch.float32:
        return SPARK_F32
    raise ValueError(f"unsupported dtype {t}")


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------------ sizes
def spark_lambda_to_T(lam: float, D: int = 128) -> int:
    return int(lib().spark_lambda_to_T(ctypes.c_float(lam), D))


def spark_cache_sizes(B, Hkv, S, D, T, dtype) -> tuple[int, list[int]]:
    sizes = (ctypes.c_size_t * 4)()
    total = lib().spark_cache_sizes(B, Hkv, S, D, T, dtype, sizes)
    return int(total), [int(x) for x in sizes]


def spark_cache_bytes(B, Hkv, S, D, T, dtype) -> int:
    return int(lib().spark_cache_bytes(B, Hkv, S, D, T, dtype))


def spark_workspace_bytes(op, B, Hkv, G, S, D, T, n_tail) -> int:
    return int(lib().spark_workspace_bytes(op, B, Hkv, G, S, D, T, n_tail))


# ------------------------------------------------------------------ cache
@dataclass
class KCache:
    """Device tensors of the packed key cache (layout of include/spark.h)."""
    B: int
    Hkv: int
    S: int
    D: int
    T: int
    dtype: torch.dtype
    mask: torch.Tensor    # uint32 bits stored as int32 [B, Hkv, S, 4]
    vals: torch.Tensor    # [B, Hkv, S32 * T] interleaved by 32-token groups
    qn: torch.Tensor      # fp32 [B, Hkv, D]
    stats: torch.Tensor   # fp64 [B, Hkv, 4]
    goff: torch.Tensor = None  # SparK-p only: int32 [B * Hkv * S32 / 32 + 1] first value row per group
    lens: torch.Tensor = None  # optional int32 [B] prompt tokens per row (S is then the row stride)

    @staticmethod
    def empty(B, Hkv, S, D, T, dtype, device="cuda") -> "KCache":
        S32 = (S + 31) // 32 * 32
        return KCache(B, Hkv, S, D, T, dtype,
                      torch.empty((B, Hkv, S, 4), dtype=torch.int32, device=device),
                      torch.empty((B, Hkv, S32 * T), dtype=dtype, device=device),
                      torch.empty((B, Hkv, D), dtype=torch.float32, device=device),
                      torch.empty((B, Hkv, 4), dtype=torch.float64, device=device))

    @staticmethod
    def empty_topp(B, Hkv, S, D, Tcap, dtype, device="cuda") -> "KCache":
        """A SparK-p cache: masks, a value stream with room for Tcap slots per
        token (the most spark_prune_topp can write) and the group offsets."""
        kc = KCache.empty(B, Hkv, S, D, Tcap, dtype, device)
        kc.vals = kc.vals.reshape(-1)
        kc.goff = torch.empty((B * Hkv * ((S + 31) // 32) + 1,), dtype=torch.int32, device=device)
        return kc

    def struct(self) -> spark_kcache:
        return spark_kcache(self.B, self.Hkv, self.S, self.D, self.T, _dtype_code(self.dtype),
                            _ptr(self.mask), _ptr(self.vals), _ptr(self.qn), _ptr(self.stats),
                            _ptr(self.goff) if self.goff is not None else None,
                            _ptr(self.lens) if self.lens is not None else None)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.mask, self.vals, self.qn, self.stats))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zero-initialised workspace (the status word must start at zero)."""
    n = (max(nbytes, 256) + 255) // 256 * 256
    return torch.zeros(n, dtype=torch.uint8, device=device)


# ------------------------------------------------------------- entry points
def spark_prune(k: torch.Tensor, q_obs: torch.Tensor, G: int, W: int, kc: KCache,
                ws: torch.Tensor, stream=None) -> None:
    s = kc.struct()
    rc = lib().spark_prune(_ptr(k), _ptr(q_obs), G, W, ctypes.byref(s), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_prune")


def spark_prune_noalloc(k: torch.Tensor, q_obs: torch.Tensor, G: int, W: int, kc: KCache,
                        stream=None) -> None:
    """spark_prune for callers that cannot allocate a workspace: the library's
    fixed 4 MiB per-device scratch array stands in for it (see spark.h)."""
    s = kc.struct()
    rc = lib().spark_prune_noalloc(_ptr(k), _ptr(q_obs), G, W, ctypes.byref(s), _stream(stream))
    _check(rc, "spark_prune_noalloc")


def spark_prune_grouped(k: torch.Tensor, q_obs: torch.Tensor, G: int, W: int, group_T, kc: KCache,
                        ws: torch.Tensor, stream=None) -> None:
    """SparK-g: per-group kept-channel budgets group_T (host list, one entry
    per group, sum == kc.T); groups by window-query norm rank (see spark.h)."""
    tg = (ctypes.c_int * len(group_T))(*[int(x) for x in group_T])
    s = kc.struct()
    rc = lib().spark_prune_grouped(_ptr(k), _ptr(q_obs), G, W, len(group_T), tg, ctypes.byref(s), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_prune_grouped")


def spark_prune_think(k: torch.Tensor, q_obs: torch.Tensor, G: int, W: int, kc: KCache, ws: torch.Tensor,
                      stream=None) -> None:
    """ThinK structured pruning (comparator): one channel mask per head (see spark.h)."""
    s = kc.struct()
    rc = lib().spark_prune_think(_ptr(k), _ptr(q_obs), G, W, ctypes.byref(s), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_prune_think")


def spark_prune_topp(k: torch.Tensor, q_obs: torch.Tensor, G: int, W: int, p: float, kc: KCache,
                     ws: torch.Tensor, stream=None) -> None:
    """SparK-p: per token the fewest greedy-order channels whose saliency mass
    reaches p of the total, at most kc.T of them (see spark.h)."""
    s = kc.struct()
    rc = lib().spark_prune_topp(_ptr(k), _ptr(q_obs), G, W, ctypes.c_float(p), ctypes.byref(s), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_prune_topp")


def spark_topp_offsets_bytes(B: int, Hkv: int, S: int) -> int:
    return int(lib().spark_topp_offsets_bytes(B, Hkv, S))


def spark_topp_vals_used(kc: KCache, stream=None) -> int:
    """Bytes of kc.vals the last spark_prune_topp used (synchronises the stream)."""
    s = kc.struct()
    n = ctypes.c_size_t(0)
    _check(lib().spark_topp_vals_used(ctypes.byref(s), ctypes.byref(n), _stream(stream)), "spark_topp_vals_used")
    return int(n.value)


def spark_decode_attn_topp(q: torch.Tensor, kc: KCache, v: torch.Tensor, k_tail, v_tail, tail_cap: int,
                           n_tail: int, G: int, out: torch.Tensor, ws: torch.Tensor,
                           recovery: int = SPARK_F_DEGENERATE, seed: int = 0, stream=None) -> None:
    """spark_decode_attn over a SparK-p cache (masks with at most kc.T bits)."""
    s = kc.struct()
    rc = lib().spark_decode_attn_topp(_ptr(q), ctypes.byref(s), _ptr(v), _ptr(k_tail), _ptr(v_tail), tail_cap,
                                      n_tail, G, recovery, seed, _ptr(out), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_decode_attn_topp")


def spark_selftest_wait_timeout(ws: torch.Tensor, limit_us: int, stream=None) -> None:
    """Make one bounded device wait run out on purpose (status word test)."""
    _check(lib().spark_selftest_wait_timeout(_ptr(ws), limit_us, _stream(stream)), "spark_selftest_wait_timeout")


def spark_prune_values(v: torch.Tensor, vc: KCache, ws: torch.Tensor, stream=None) -> None:
    """Value-channel pruning: top-vc.T channels of |v| per token (see spark.h)."""
    s = vc.struct()
    rc = lib().spark_prune_values(_ptr(v), ctypes.byref(s), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream))
    _check(rc, "spark_prune_values")


def spark_decode_attn_kv(q: torch.Tensor, kc: KCache, vc: KCache, k_tail, v_tail, tail_cap: int, n_tail: int,
                         G: int, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    sk, sv = kc.struct(), vc.struct()
    rc = lib().spark_decode_attn_kv(_ptr(q), ctypes.byref(sk), ctypes.byref(sv), _ptr(k_tail), _ptr(v_tail),
                                    tail_cap, n_tail, G, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(stream))
    _check(rc, "spark_decode_attn_kv")


def spark_workspace_bytes_kv(B: int, Hkv: int, G: int, S: int, D: int, T: int, Tv: int, n_tail: int) -> int:
    return int(lib().spark_workspace_bytes_kv(B, Hkv, G, S, D, T, Tv, n_tail))


def spark_group_budget(D: int, rates) -> list:
    """Per-group kept-channel budgets of SparK-g (the C library's
    spark_group_budget): round((1 - rate) * group size), half away from zero,
    for len(rates) equal-rank groups of D channels."""
    g = len(rates)
    arr = (ctypes.c_float * max(g, 1))(*[float(r) for r in rates])
    out = (ctypes.c_int * max(g, 1))()
    _check(lib().spark_group_budget(D, g, arr, out), "spark_group_budget")
    return [int(out[q]) for q in range(g)]


def spark_decode_attn(q: torch.Tensor, kc: KCache, v: torch.Tensor, k_tail, v_tail, tail_cap: int,
                      n_tail: int, G: int, out: torch.Tensor, ws: torch.Tensor,
                      recovery: int = SPARK_F_DEGENERATE, seed: int = 0, stream=None) -> None:
    s = kc.struct()
    rc = lib().spark_decode_attn(_ptr(q), ctypes.byref(s), _ptr(v), _ptr(k_tail), _ptr(v_tail), tail_cap,
                                 n_tail, G, recovery, seed, _ptr(out), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_decode_attn")


def spark_snapkv_evict(k: torch.Tensor, v: torch.Tensor, q_obs: torch.Tensor, G: int, W: int, keep: int,
                       pool: int, k_out: torch.Tensor, v_out: torch.Tensor, idx_out: torch.Tensor,
                       ws: torch.Tensor, stream=None) -> None:
    """SnapKV-style eviction: k, v [B, Hkv, S, D] -> k_out, v_out [B, Hkv, keep, D],
    idx_out int32 [B, Hkv, keep]."""
    B, H, S, D = k.shape
    rc = lib().spark_snapkv_evict(_ptr(k), _ptr(v), _ptr(q_obs), B, H, S, D, G, W, keep, pool,
                                  _dtype_code(k.dtype), _ptr(k_out), _ptr(v_out), _ptr(idx_out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_snapkv_evict")


def spark_snapkv_evict_rows(k: torch.Tensor, v: torch.Tensor, q_obs: torch.Tensor, G: int, W: int,
                            keep_rows: torch.Tensor, keep_cap: int, pool: int, k_out: torch.Tensor,
                            v_out: torch.Tensor, idx_out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """SnapKV-style eviction with one budget per row (keep_rows: int32 [B] on
    the device); outputs with row stride keep_cap (see spark.h)."""
    B, Hkv, S, D = k.shape
    rc = lib().spark_snapkv_evict_rows(_ptr(k), _ptr(v), _ptr(q_obs), B, Hkv, S, D, G, W, _ptr(keep_rows),
                                       keep_cap, pool, _dtype_code(k.dtype), _ptr(k_out), _ptr(v_out),
                                       _ptr(idx_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "spark_snapkv_evict_rows")


def spark_pyramid_keep(L: int, M: int, beta: float, W: int, S: int) -> list:
    """PyramidKV-style layer budgets around the mean M (the library's linear
    reading, see spark.h)."""
    out = (ctypes.c_int * max(L, 1))()
    _check(lib().spark_pyramid_keep(L, M, ctypes.c_float(beta), W, S, out), "spark_pyramid_keep")
    return [int(out[i]) for i in range(L)]


def spark_tail_append(k_new, v_new, k_tail, v_tail, B, Hkv, D, tail_cap, slot, stream=None) -> None:
    rc = lib().spark_tail_append(_ptr(k_new), _ptr(v_new), _ptr(k_tail), _ptr(v_tail), B, Hkv, D,
                                 tail_cap, slot, _dtype_code(k_new.dtype), _stream(stream))
    _check(rc, "spark_tail_append")


def spark_device_status(ws: torch.Tensor, clear: bool = False, stream=None) -> int:
    st = ctypes.c_int(0)
    rc = lib().spark_device_status(_ptr(ws), ctypes.byref(st), int(clear), _stream(stream))
    _check(rc, "spark_device_status")
    return st.value
