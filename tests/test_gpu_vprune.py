"""GPU parity of value-channel pruning (spark_prune_values) and of decode over
pruned key and value caches (spark_decode_attn_kv) against the oracle's
prune_values / decode_kv on the same seeded inputs: value masks and kept
values bit for bit (near-ties counted, < 0.01 %), attention outputs within
max-abs 2e-3 and relative 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_decode_attn_kv, spark_device_status, spark_prune_values,
                                        spark_tail_append, spark_workspace_bytes, spark_workspace_bytes_kv,
                                        workspace, SPARK_OP_PRUNE)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, compare_masks, mask_np, run_prune, to_np, unpack_vals

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


def run_prune_values(v, Tv):
    R, Hkv, S, _ = v.shape
    vc = KCache.empty(R, Hkv, S, D, Tv, v.dtype, device=v.device)
    ws = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, Hkv, 1, S, D, Tv, 0))
    spark_prune_values(v, vc, ws)
    torch.cuda.synchronize()
    return vc


def check_values(vc, v_np, Tv, what):
    BH, S = vc.B * vc.Hkv, vc.S
    v3 = v_np.reshape(BH, S, D)
    vm_o, vv_o, _ = oracle.prune_values(v3, Tv)
    vm_g = mask_np(vc)
    rep = compare_masks(vm_g, vm_o, v3, np.ones((BH, D), np.float32), Tv)
    assert rep["mismatch"] == rep["near_tie"] and rep["mismatch"] <= max(1e-4 * rep["tokens"], 0), (what, rep)
    ok = np.all(vm_g == vm_o, axis=-1)
    assert np.array_equal(unpack_vals(vc)[ok].view(np.uint32), vv_o[ok].view(np.uint32)), what
    assert np.all(vc.qn.cpu().numpy() == 1.0)
    return vm_o, vv_o


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S,Tv", [(1, 64), (33, 0), (1000, 64), (257, 128), (2049, 13), (0, 64)])
def test_prune_values_parity(dtype, S, Tv):
    wl = scaled(WORKLOADS["tiny"], S=S, Hkv=3, dtype="f32" if dtype == torch.float32 else "bf16", seed=90 + S)
    pre = make_prefill(wl, DEV)
    vc = run_prune_values(pre["v"], Tv)
    check_values(vc, to_np(pre["v"]), Tv, f"values S={S} Tv={Tv}")


def _decode_kv(q, kc, vc, kt, vt, cap, n_tail, G):
    R, Hq, _ = q.shape
    out = torch.empty((R, Hq, D), dtype=torch.float32, device=DEV)
    ws = workspace(spark_workspace_bytes_kv(kc.B, kc.Hkv, G, kc.S, D, kc.T, vc.T, cap))
    spark_decode_attn_kv(q, kc, vc, kt, vt, cap, n_tail, G, out, ws)
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    return out


@pytest.mark.parametrize("S,T,Tv,G,n_tail", [(1, 26, 64, 4, 0), (33, 26, 64, 4, 3), (1000, 64, 64, 4, 0),
                                             (777, 26, 0, 2, 5), (640, 90, 128, 1, 0), (129, 64, 38, 8, 64),
                                             (0, 26, 64, 4, 7), (2049, 26, 26, 4, 256)])
def test_decode_kv_parity(S, T, Tv, G, n_tail):
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, Hkv=3, dtype="bf16", seed=5 + S + T + Tv)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], G, wl.W, T)
    vc = run_prune_values(pre["v"], Tv)
    torch.cuda.synchronize()
    BH = wl.rows * wl.Hkv
    k_np, q_np = to_np(pre["k"]).reshape(BH, S, D), to_np(pre["q_obs"]).reshape(BH * G, -1, D)
    qn = oracle.qnorm(q_np, G)
    m, vals, st = oracle.prune(k_np, qn, T)
    vm, vv = check_values(vc, to_np(pre["v"]), Tv, f"values S={S}")
    cap = max(n_tail, 8)
    kt = torch.zeros((wl.rows, wl.Hkv, cap, D), dtype=torch.bfloat16, device=DEV)
    vt = torch.zeros_like(kt)
    for i in range(n_tail):
        stp = make_decode_step(wl, i, DEV)
        spark_tail_append(stp["k_new"], stp["v_new"], kt, vt, wl.rows, wl.Hkv, D, cap, i)
    q = make_decode_step(wl, 77, DEV)["q"]
    out = _decode_kv(q, kc, vc, kt, vt, cap, n_tail, G)
    ok = np.all(mask_np(kc) == m, axis=-1).all() and np.all(mask_np(vc) == vm, axis=-1).all()
    assert ok, "masks differ from the oracle (near-ties): decode comparison needs identical caches"
    o_ref = oracle.decode_kv(to_np(q).reshape(BH * G, D), m, vals, qn, st, vm, vv, to_np(kt).reshape(BH, cap, D),
                             to_np(vt).reshape(BH, cap, D), n_tail, G)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"decode_kv S={S} T={T} Tv={Tv} G={G}")


def test_decode_kv_lambda_05_05_sampled_heads():
    # the pages' SparK(0.5 + 0.5): half of the key and half of the value
    # channels pruned, on the lambda-sweep shape (B=8, S=16384); the oracle
    # checks a sample of heads
    wl = WORKLOADS["lsweep_0.5"]
    pre = make_prefill(wl, DEV)
    T = Tv = 64
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
    vc = run_prune_values(pre["v"], Tv)
    q = make_decode_step(wl, 3, DEV)["q"]
    out = _decode_kv(q, kc, vc, None, None, 0, 0, wl.G)
    sel = [0, 9, 33, 63]
    k_np = to_np(pre["k"].reshape(wl.BH, wl.S, D)[sel])
    v_np = to_np(pre["v"].reshape(wl.BH, wl.S, D)[sel])
    qsel = np.concatenate([np.arange(b * wl.G, (b + 1) * wl.G) for b in sel])
    q_obs = to_np(pre["q_obs"].reshape(wl.BH * wl.G, wl.W, D)[torch.as_tensor(qsel, device=DEV)])
    qn = oracle.qnorm(q_obs, wl.G)
    m, vals, st = oracle.prune(k_np, qn, T)
    vm, vv, _ = oracle.prune_values(v_np, Tv)
    assert np.array_equal(mask_np(kc)[sel], m) and np.array_equal(mask_np(vc)[sel], vm)
    o_ref = oracle.decode_kv(to_np(q).reshape(wl.BH * wl.G, D)[qsel], m, vals, qn, st, vm, vv, G=wl.G)
    assert_out_close(out.cpu().numpy().reshape(wl.BH * wl.G, D)[qsel], o_ref, "SparK(0.5+0.5)")
