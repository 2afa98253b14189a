"""Seeded synthetic inputs shaped like the SparK pages' Llama-3.1 workloads.

This module holds no pruning or attention arithmetic: it only draws random
tensors.  Both the CUDA path and the CPU oracle are fed from it.

Recipe (the pages run LLaMA3-8B / LLaMA3.1-8B on LongBench and RULER; no
weights or datasets are available, so these shapes and distributions stand
in for them):

* every key / value / query element is x = z * s_c, z ~ N(0, 1), with a
  per-channel outlier scale s_c ~ LogNormal(0, 1) drawn once per
  (layer, head, channel) and shared by all tokens and batch rows;
  keys and values use per-kv-head scales, queries per-query-head scales;
* drawn in fp32 and rounded to the workload dtype (bf16 round-to-nearest-even,
  or kept fp32 for the tiny parity case);
* decode-step queries and appended keys/values use the same scales, with a
  generator seeded per step so any step can be regenerated on its own.

Flattened batch: rows are ordered (layer, batch), i.e. row = l * B + b, so a
layer's rows are contiguous.  Query head g of kv head h is h * G + g.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    Hkv: int
    G: int
    S: int
    D: int
    W: int
    lam: float
    dtype: str  # "f32" | "bf16"
    steps: int
    seed: int
    keep: int = 0      # SnapKV keep budget per head (0: no eviction pre-pass)
    pool: int = 7      # SnapKV max-pool kernel
    tail_cap: int = 256

    @property
    def BH(self) -> int:
        return self.L * self.B * self.Hkv

    @property
    def rows(self) -> int:
        return self.L * self.B

    @property
    def Hq(self) -> int:
        return self.Hkv * self.G

    @property
    def S_kept(self) -> int:
        return self.keep if self.keep else self.S

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    # tiny parity case: B1, 1 layer, 2 kv heads x group 4, S=512, fp32, W=16
    "tiny": Workload("tiny", 1, 1, 2, 4, 512, 128, 16, 0.5, "f32", 1, 0),
    # Llama-3.1-8B single layer, S=32768, lambda 0.5, 64 decode steps
    "llama1l": Workload("llama1l", 1, 1, 8, 4, 32768, 128, 32, 0.5, "bf16", 64, 1),
    # lambda sweep, B=8, S=16384, 128 decode steps
    "lsweep_0.3": Workload("lsweep_0.3", 8, 1, 8, 4, 16384, 128, 32, 0.3, "bf16", 128, 2),
    "lsweep_0.5": Workload("lsweep_0.5", 8, 1, 8, 4, 16384, 128, 32, 0.5, "bf16", 128, 3),
    "lsweep_0.8": Workload("lsweep_0.8", 8, 1, 8, 4, 16384, 128, 32, 0.8, "bf16", 128, 4),
    # long context: 32 layers x 8 kv heads, S=131072, lambda 0.8, one decode step
    "long": Workload("long", 1, 32, 8, 4, 131072, 128, 32, 0.8, "bf16", 1, 5),
    # stacked with SnapKV-style eviction: keep 2048 of 8192, then lambda 0.5
    "evict": Workload("evict", 32, 1, 8, 4, 8192, 128, 32, 0.5, "bf16", 256, 6,
                      keep=2048, pool=7),
}


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return replace(wl, **kw)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _lognormal(gen, shape, device):
    return torch.exp(torch.randn(shape, generator=gen, device=device, dtype=torch.float32))


def channel_scales(wl: Workload, device="cpu"):
    """Per-(layer, head, channel) LogNormal(0,1) outlier scales for k, v, q."""
    gen = _gen(device, wl.seed * 7919 + 11)
    s_k = _lognormal(gen, (wl.L, wl.Hkv, wl.D), device)
    s_v = _lognormal(gen, (wl.L, wl.Hkv, wl.D), device)
    s_q = _lognormal(gen, (wl.L, wl.Hq, wl.D), device)
    return s_k, s_v, s_q


def _draw(gen, shape, scale, dtype, device):
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return (z * scale).to(dtype)


def make_prefill(wl: Workload, device="cpu", scales=None):
    """Prompt keys/values and observation-window queries.

    Returns dict with k, v: [L*B, Hkv, S, D]; q_obs: [L*B, Hq, W, D]
    in the workload dtype.  Drawn one layer at a time so the fp32
    temporaries stay one layer large."""
    s_k, s_v, s_q = scales if scales is not None else channel_scales(wl, device)
    dt = wl.torch_dtype
    R = wl.rows
    k = torch.empty((R, wl.Hkv, wl.S, wl.D), dtype=dt, device=device)
    v = torch.empty_like(k)
    q_obs = torch.empty((R, wl.Hq, wl.W, wl.D), dtype=dt, device=device)
    for l in range(wl.L):
        gen = _gen(device, wl.seed * 1000003 + 17 * l + 1)
        sl = slice(l * wl.B, (l + 1) * wl.B)
        k[sl] = _draw(gen, (wl.B, wl.Hkv, wl.S, wl.D), s_k[l][None, :, None, :], dt, device)
        v[sl] = _draw(gen, (wl.B, wl.Hkv, wl.S, wl.D), s_v[l][None, :, None, :], dt, device)
        q_obs[sl] = _draw(gen, (wl.B, wl.Hq, wl.W, wl.D), s_q[l][None, :, None, :], dt, device)
    return {"k": k, "v": v, "q_obs": q_obs}


def make_decode_step(wl: Workload, step: int, device="cpu", scales=None):
    """Query of decode step `step` and the unpruned key/value it appends.

    Returns dict with q: [L*B, Hq, D]; k_new, v_new: [L*B, Hkv, D]."""
    s_k, s_v, s_q = scales if scales is not None else channel_scales(wl, device)
    dt = wl.torch_dtype
    gen = _gen(device, wl.seed * 1000003 + 500009 + 31 * step)
    R = wl.rows
    q = torch.empty((R, wl.Hq, wl.D), dtype=dt, device=device)
    k_new = torch.empty((R, wl.Hkv, wl.D), dtype=dt, device=device)
    v_new = torch.empty_like(k_new)
    for l in range(wl.L):
        sl = slice(l * wl.B, (l + 1) * wl.B)
        q[sl] = _draw(gen, (wl.B, wl.Hq, wl.D), s_q[l][None], dt, device)
        k_new[sl] = _draw(gen, (wl.B, wl.Hkv, wl.D), s_k[l][None], dt, device)
        v_new[sl] = _draw(gen, (wl.B, wl.Hkv, wl.D), s_v[l][None], dt, device)
    return {"q": q, "k_new": k_new, "v_new": v_new}
