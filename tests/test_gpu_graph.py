"""The decode loop of a serving step (append the new key/value to the dense
tail, then decode) is launch-bound at small batch: capturing a sequence of
such steps in one CUDA graph and replaying it must give exactly the outputs
of the same calls made one by one (same kernels, same arguments), and the
last step must match the oracle."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (spark_decode_attn, spark_device_status, spark_lambda_to_T,
                                        spark_tail_append, spark_workspace_bytes, workspace, SPARK_OP_DECODE)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, mask_np, run_prune, to_np, unpack_vals

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


def test_decode_loop_replayed_from_a_cuda_graph():
    wl = scaled(WORKLOADS["llama1l"], S=8192)
    T = spark_lambda_to_T(wl.lam)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
    R, H, G = wl.rows, wl.Hkv, wl.G
    steps, cap = 12, 16
    st = [make_decode_step(wl, i, DEV) for i in range(steps)]
    kt = torch.zeros((R, H, cap, D), dtype=wl.torch_dtype, device=DEV)
    vt = torch.zeros_like(kt)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, R, H, G, wl.S, D, T, cap))
    outs = [torch.empty((R, H * G, D), dtype=torch.float32, device=DEV) for _ in range(2 * steps)]

    def run(out_base, stream=None):
        for i in range(steps):
            spark_tail_append(st[i]["k_new"], st[i]["v_new"], kt, vt, R, H, D, cap, i, stream)
            spark_decode_attn(st[i]["q"], kc, pre["v"], kt, vt, cap, i + 1, G, outs[out_base + i], ws,
                              stream=stream)

    run(0)  # eager, one call at a time
    torch.cuda.synchronize()
    kt.zero_()
    vt.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run(steps)
    torch.cuda.synchronize()
    kt.zero_()
    vt.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    for i in range(steps):
        assert torch.equal(outs[i], outs[steps + i]), f"step {i}"
    # the last step against the oracle
    BH = R * H
    qn = oracle.qnorm(to_np(pre["q_obs"]).reshape(BH * G, -1, D), G)
    m, vals, stt = oracle.prune(to_np(pre["k"]).reshape(BH, wl.S, D), qn, T)
    ref = oracle.decode(to_np(st[-1]["q"]).reshape(BH * G, D), m, vals, qn, stt,
                        to_np(pre["v"]).reshape(BH, wl.S, D), to_np(kt).reshape(BH, cap, D),
                        to_np(vt).reshape(BH, cap, D), steps, G)
    assert_out_close(outs[2 * steps - 1].cpu().numpy().reshape(BH * G, D), ref, "graph replay last step")
    del g
