"""Benchmark of the SparK hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
window-norm + top-T channel pruning + pruned-saliency statistics over every
(layer, kv head) of the prompt (spark_prune), one unpruned key/value appended
to the dense tail (spark_tail_append), and one decode-attention step over the
pruned cache plus tail for every layer (spark_decode_attn: split-K kernel and
log-sum-exp combine).  Default workload: the pages' long-context Llama-3.1-8B
shape -- B=1, 32 layers x 8 kv heads x GQA 4, D=128, S=131072, bf16,
lambda=0.8 (T=26).

Prints ONE JSON line (rank 0).  `--impl reference` times the CPU oracle (the
only reference this method has) on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from channel_pruned_decode_b200 import dist as sd  # noqa: E402
from channel_pruned_decode_b200.synth import (WORKLOADS, make_decode_step, make_prefill,  # noqa: E402
                                              scaled)

METRIC = "decode-attn KV tokens·heads/s & HBM GB/s (frac of 8 TB/s); spark_prune GB/s"
UNIT = "KV token·heads/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _workload_desc(wl, T):
    return (f"{wl.name}: B={wl.B} L={wl.L} Hkv={wl.Hkv} G={wl.G} S={wl.S} D={wl.D} W={wl.W} "
            f"lambda={wl.lam} (T={T}) {wl.dtype}; prune all layers + tail append + 1 decode step")


def _byte_model(wl, T, n_tail):
    """Algorithmic HBM bytes per launch of the two heavy calls (on the
    prompt as it stands after any eviction)."""
    es = 2 if wl.dtype == "bf16" else 4
    BH, S, D, G = wl.BH, wl.S_kept, wl.D, wl.G
    prune = BH * S * (D * es + 16 + T * es) + BH * G * wl.W * D * es + BH * (D * 4 + 32)
    decode = (BH * S * (16 + T * es + D * es) + BH * n_tail * 2 * D * es
              + BH * G * D * (es + 4) + BH * (D * 4 + 32))
    out = {"prune": prune, "decode": decode, "per_token_head_prune": D * es + 16 + T * es,
           "per_token_head_decode": 16 + T * es + D * es}
    if wl.keep:
        # eviction: the keys read once for the scores, the window queries,
        # the kept K and V rows read and written, the kept indices written
        S0 = wl.S
        out["snapkv"] = (BH * S0 * D * es + BH * G * wl.W * D * es + 4 * BH * wl.keep * D * es
                         + BH * wl.keep * 4)
    return out


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            bus = torch.cuda.get_device_properties(device_index).pci_bus_id
            dom, rest = bus.split(":", 1)
            bus = dom.zfill(8) + ":" + rest  # nvidia-smi's 8-digit PCI domain form
        except Exception:
            bus = str(device_index)
        self.bus = bus

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# -------------------------------------------------------------- GPU arm
class Job:
    """Device buffers and the step of one rank."""

    def __init__(self, wl, dev, host_inputs: bool = False):
        import channel_pruned_decode_b200 as sp
        self.sp = sp
        self.wl = wl
        self.dev = dev
        self.T = sp.spark_lambda_to_T(wl.lam, wl.D)
        pre = make_prefill(wl, dev)
        self.k, self.v, self.q_obs = pre["k"], pre["v"], pre["q_obs"]
        stp = make_decode_step(wl, 0, dev)
        self.q, self.k_new, self.v_new = stp["q"], stp["k_new"], stp["v_new"]
        R, H, S, D, G = wl.rows, wl.Hkv, wl.S, wl.D, wl.G
        self.cap = wl.tail_cap
        self.kt = torch.zeros((R, H, self.cap, D), dtype=wl.torch_dtype, device=dev)
        self.vt = torch.zeros_like(self.kt)
        self.kc = sp.KCache.empty(R, H, S, D, self.T, wl.torch_dtype, device=dev)
        self.wsp = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_PRUNE, R, H, G, S, D, self.T, 0), dev)
        self.wsd = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_DECODE, R, H, G, S, D, self.T,
                                                         self.cap), dev)
        self.out = torch.empty((R, wl.Hq, D), dtype=torch.float32, device=dev)
        self.n_tail = 0
        self.launches_per_step = 6  # qnorm, prune, stats, tail append, decode, combine
        self.S_kept = S
        if wl.keep:
            # SnapKV-style eviction first: the cache then holds `keep` tokens
            self.S_kept = wl.keep
            self.k_ev = torch.empty((R, H, wl.keep, D), dtype=wl.torch_dtype, device=dev)
            self.v_ev = torch.empty_like(self.k_ev)
            self.idx = torch.empty((R, H, wl.keep), dtype=torch.int32, device=dev)
            self.wse = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_SNAPKV, R, H, G, S, D, 0, 0), dev)
            self.kc = sp.KCache.empty(R, H, wl.keep, D, self.T, wl.torch_dtype, device=dev)
            self.wsp = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_PRUNE, R, H, G, wl.keep, D, self.T, 0), dev)
            self.wsd = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_DECODE, R, H, G, wl.keep, D, self.T,
                                                             self.cap), dev)
            self.launches_per_step += 4  # two score passes, select, gather

    def step(self, stream, ev=None):
        sp, wl = self.sp, self.wl
        slot = 0  # one decode step per bench step: the tail holds this step's token
        k, v = self.k, self.v
        if ev is not None:
            ev[4].record(stream)
        if wl.keep:
            sp.spark_snapkv_evict(self.k, self.v, self.q_obs, wl.G, wl.W, wl.keep, wl.pool, self.k_ev, self.v_ev,
                                  self.idx, self.wse, stream)
            k, v = self.k_ev, self.v_ev
        if ev is not None:
            ev[0].record(stream)
        sp.spark_prune(k, self.q_obs, wl.G, wl.W, self.kc, self.wsp, stream)
        if ev is not None:
            ev[1].record(stream)
        sp.spark_tail_append(self.k_new, self.v_new, self.kt, self.vt, wl.rows, wl.Hkv, wl.D, self.cap,
                             slot, stream)
        if ev is not None:
            ev[2].record(stream)
        sp.spark_decode_attn(self.q, self.kc, v, self.kt, self.vt, self.cap, slot + 1, wl.G,
                             self.out, self.wsd, stream=stream)
        if ev is not None:
            ev[3].record(stream)


def _barrier(dist_on):
    sd.barrier()


def _max_over_ranks(x: float, dist_on: bool) -> float:
    return sd.max_over_ranks(x, device="cuda") if dist_on else float(x)


def _traffic_record(kernel: str, workload: str):
    """The committed ncu record of a kernel (DRAM bytes per launch, issue and
    pipe counters), if it was taken on the current source of the kernel
    (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            recs = json.load(f)
    except Exception:
        return None
    rec = recs.get(f"{kernel}@{workload}")
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except Exception:
        return None
    return rec if h == rec["source_sha"] else None


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(wl, job, units: int | None = None):
    """The CPU oracle, as it stands, on a bounded sample of the workload:
    prune + decode (with the step's one-token tail) of whole (layer, kv head)
    units, threads over units; the same oracle outputs then check the GPU's
    results for those units (sampled parity)."""
    import concurrent.futures as cf

    import numpy as np

    import oracle

    lib = oracle.load()
    BH, D, G = wl.BH, wl.D, wl.G
    S = job.S_kept  # the tokens the GPU pruned (after eviction, if any)
    cores = os.cpu_count() or 1
    units = units or min(BH, cores)
    sel = list(range(0, BH, max(1, BH // units)))[:units]
    # one untimed GPU step, so that the cache, the tail and the output hold
    # this step's results whatever ran before
    stream = torch.cuda.current_stream()
    job.step(stream)
    torch.cuda.synchronize()
    k_src, v_src = (job.k_ev, job.v_ev) if wl.keep else (job.k, job.v)
    k = k_src.reshape(BH, S, D)
    v = v_src.reshape(BH, S, D)
    kt = job.kt.reshape(BH, job.cap, D)
    vt = job.vt.reshape(BH, job.cap, D)
    qo = job.q_obs.reshape(BH * G, wl.W, D)
    q = job.q.reshape(BH * G, D)
    data = []
    for b in sel:
        data.append((k[b:b + 1].float().cpu().numpy(), v[b:b + 1].float().cpu().numpy(),
                     qo[b * G:(b + 1) * G].float().cpu().numpy(), q[b * G:(b + 1) * G].float().cpu().numpy(),
                     kt[b:b + 1].float().cpu().numpy(), vt[b:b + 1].float().cpu().numpy()))

    def prune_one(d):
        kk, vv, qq, q1, kt1, vt1 = d
        qn = oracle.qnorm(qq, G, lib=lib)
        return qn, oracle.prune(kk, qn, job.T, lib=lib)

    def decode_one(d, pr):
        kk, vv, qq, q1, kt1, vt1 = d
        qn, (m, vals, st) = pr
        return oracle.decode(q1, m, vals, qn, st, vv, kt1, vt1, 1, G=G, lib=lib)

    # one unit on one thread, then the sample on the pool, prune and decode
    # timed as separate phases
    t0 = time.perf_counter()
    decode_one(data[0], prune_one(data[0]))
    single = time.perf_counter() - t0
    with cf.ThreadPoolExecutor(max_workers=min(cores, len(data))) as ex:
        t0 = time.perf_counter()
        prs = list(ex.map(prune_one, data))
        t1 = time.perf_counter()
        outs = list(ex.map(decode_one, data, prs))
        t2 = time.perf_counter()
    dt = t2 - t0
    return {"value": len(data) * S / dt, "unit": UNIT, "cores": min(cores, len(data)), "kind": "oracle",
            "sample": f"{len(data)} of {BH} (layer, kv head) units, full S={S}"
                      f"{' (the tokens kept by the GPU eviction)' if wl.keep else ''}: prune + 1 decode step "
                      f"with the one-token tail, {dt:.1f} s wall",
            "prune_s": t1 - t0, "decode_s": t2 - t1, "single_thread_unit_s": single,
            "cpu_model": _cpu_model(), "parity": _sample_parity(job, sel, prs, outs, S)}


def _sample_parity(job, sel, prs, outs, S):
    """The GPU's cache and decode output of the sampled units against the
    oracle's: tokens whose mask differs, tokens whose packed values differ,
    the largest relative error of the statistics, the largest absolute error
    of the decode output."""
    import numpy as np

    BH, G, D, T = job.wl.BH, job.wl.G, job.wl.D, job.T
    st = torch.as_tensor(sel, device=job.kc.mask.device)
    m_g = job.kc.mask.reshape(BH, S, 4)[st].cpu().numpy().view(np.uint32)
    S32 = (S + 31) // 32 * 32
    v_g = (job.kc.vals.reshape(BH, S32 // 32, T, 32)[st].float().permute(0, 1, 3, 2)
           .reshape(len(sel), S32, T)[:, :S].cpu().numpy()) if T > 0 else np.zeros((len(sel), S, 0), np.float32)
    s_g = job.kc.stats.reshape(BH, 4)[st].cpu().numpy()
    rows = torch.as_tensor(np.concatenate([np.arange(b * G, (b + 1) * G) for b in sel]), device=job.out.device)
    o_g = job.out.reshape(BH * G, D)[rows].cpu().numpy().reshape(len(sel), G, D)
    mask_bad = vals_bad = 0
    stats_rel = out_abs = ref_abs = 0.0
    for i, ((qn, (m_o, v_o, s_o)), o_o) in enumerate(zip(prs, outs)):
        same = np.all(m_g[i] == m_o[0], axis=-1)
        mask_bad += int((~same).sum())
        vals_bad += int((~np.all(v_g[i][same] == v_o[0][same], axis=-1)).sum())
        den = np.maximum(np.abs(s_o[0, 1:3]), 1e-300)
        stats_rel = max(stats_rel, float(np.max(np.abs(s_g[i, 1:3] - s_o[0, 1:3]) / den)))
        out_abs = max(out_abs, float(np.max(np.abs(o_g[i].astype(np.float64) - o_o.reshape(G, D)))))
        ref_abs = max(ref_abs, float(np.max(np.abs(o_o))))
    return {"units": len(sel), "tokens": len(sel) * S, "mask_mismatch_tokens": mask_bad,
            "vals_mismatch_tokens": vals_bad, "stats_max_rel_err": stats_rel,
            "decode_max_abs_err": out_abs, "decode_max_abs_ref": ref_abs}


def run_gpu(args):
    dist_on = args.gpus > 1
    # one process per GPU; every rank runs its own replica of the workload
    # (independent (layer, batch, head) units: no data-path collective)
    if dist_on:
        rank, world = sd.init("nccl")
    else:
        rank, world = 0, 1
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = WORKLOADS[args.workload]
    if args.layers:
        wl = scaled(wl, L=args.layers)
    job = Job(wl, dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            job.step(stream)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    _barrier(dist_on)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            job.step(stream, evs[i])
        end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    _barrier(dist_on)
    ms_local = start.elapsed_time(end)
    prune_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    decode_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    append_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    evict_ms = sum(e[4].elapsed_time(e[0]) for e in evs) / args.steps
    ms = _max_over_ranks(ms_local, dist_on)
    st = job.sp.spark_device_status(job.wsd)
    st |= job.sp.spark_device_status(job.wsp)
    if st != 0:
        raise RuntimeError(f"device status {st} after timed region")

    token_heads = wl.BH * (wl.S_kept + 1)
    ms_per_step = ms / args.steps
    value = world * token_heads / (ms_per_step / 1e3)
    bm = _byte_model(wl, job.T, 1)
    peak, peak_kind = _peaks()
    prune_gbs = bm["prune"] / (prune_ms / 1e3) / 1e9
    decode_gbs = bm["decode"] / (decode_ms / 1e3) / 1e9
    spans = {"prune": prune_ms, "decode": decode_ms}
    if wl.keep:
        spans["snapkv"] = evict_ms
    dom = max(spans, key=spans.get)
    dom_ms = spans[dom]
    achieved = bm[dom] / (dom_ms / 1e3) / 1e9
    kernel_name = {"prune": "prune_kernel", "decode": "decode_kernel", "snapkv": "snap_tc_kernel"}[dom]
    rec = _traffic_record(kernel_name, wl.name) if dom != "snapkv" else None
    traffic = rec["bytes_per_launch"] if rec else None
    # what bounds the kernel, from the same capture: the HBM fraction above
    # is the roofline; these say which on-chip resource is the limit instead
    limiter = ({"source": "ncu --set full of the same kernel source (" + rec["captured_on"] + ")",
                **rec.get("ncu_counters", {})} if rec else None)
    timing = {"prune": "CUDA events around spark_prune on its stream (qnorm and stats, the two small "
                       "kernels launched with it, included)",
              "decode": "CUDA events around spark_decode_attn on its stream (the combine kernel "
                        "launched with it included)",
              "snapkv": "CUDA events around spark_snapkv_evict on its stream: both score passes, the "
                        "select and the gather (the bytes are those of the whole entry point)"}[dom]

    # decode alone, called back to back for ~0.6 s (sustained load: the
    # power cap may engage, unlike inside the step where decode alternates
    # with the ALU-bound prune)
    sustained = run_decode_sustained(job, wl, stream, bm["decode"], peak, peak_kind) if rank == 0 else None

    variants = None
    if not args.no_variants:
        variants = run_variants(job, wl, stream, peak, peak_kind)

    e2e = None
    if not args.no_e2e:  # every rank: the e2e timing has its own barrier and max
        e2e = run_e2e(job, wl, min(args.steps, args.e2e_steps), dist_on, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, job)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT,
            # the metric's own quantities, per step of the same timed region:
            # the decode-attention call alone and the prune call alone
            "decode_token_heads_per_s": world * token_heads / (decode_ms / 1e3),
            "decode_us": decode_ms * 1e3, "decode_gbs": decode_gbs,
            "decode_frac_8tbs": decode_gbs / NOMINAL_HBM_GBS, f"decode_frac_{peak_kind}": decode_gbs / peak,
            "prune_gbs": prune_gbs, f"prune_frac_{peak_kind}": prune_gbs / peak,
            "value_is": "whole-step throughput: prompt token-heads (+ the tail token) per second of prune + "
                        "tail append + decode",
            "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,1) x per-channel LogNormal(0,1) outlier scales)",
            "config": {"workload": _workload_desc(wl, job.T), "B": wl.B, "layers": wl.L, "Hkv": wl.Hkv,
                       "G": wl.G, "S": wl.S, "D": wl.D, "W": wl.W, "lambda": wl.lam, "T": job.T,
                       "parallelism": f"replicas x{world} (independent (layer, head) work per GPU)",
                       "l2": f"inputs (K, V: {2 * wl.BH * wl.S * wl.D * (2 if wl.dtype == 'bf16' else 4) / 1e9:.1f} GB) "
                             "exceed the 126 MB L2; no flush needed"},
            "decode": {"us_per_step": decode_ms * 1e3, "gbs": decode_gbs,
                       "frac_8tbs": decode_gbs / NOMINAL_HBM_GBS, f"frac_{peak_kind}": decode_gbs / peak,
                       "token_heads_per_s": world * token_heads / (decode_ms / 1e3),
                       "bytes_per_step": bm["decode"]},
            "prune": {"us_per_step": prune_ms * 1e3, "gbs": prune_gbs, "frac_8tbs": prune_gbs / NOMINAL_HBM_GBS,
                      f"frac_{peak_kind}": prune_gbs / peak, "bytes_per_step": bm["prune"]},
            "tail_append_us": append_ms * 1e3,
            "snapkv_evict_us": evict_ms * 1e3 if wl.keep else None,
            "snapkv": ({"us_per_step": evict_ms * 1e3, "gbs": bm["snapkv"] / (evict_ms / 1e3) / 1e9,
                        f"frac_{peak_kind}": bm["snapkv"] / (evict_ms / 1e3) / 1e9 / peak,
                        "bytes_per_step": bm["snapkv"]} if wl.keep else None),
            "roofline": {"kernel": kernel_name, "bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "limiter": limiter,
                         "traffic_source": ("committed ncu capture of the same kernel source "
                                            "(profiles/traffic.json), not measured in this run") if rec else None,
                         "bytes_per_launch": bm[dom], "entry": {"prune": "spark_prune",
                                                                "decode": "spark_decode_attn",
                                                                "snapkv": "spark_snapkv_evict"}[dom],
                         "timing": timing},
            "decode_sustained": sustained,
            "variants": variants,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": job.launches_per_step * args.steps,
        }
        print(json.dumps(line), flush=True)
    sd.finalize()


def run_decode_sustained(job, wl, stream, nbytes, peak, peak_kind, seconds=0.6):
    """spark_decode_attn alone, back to back for about `seconds` of device
    time on the launching stream (after the timed step loop), with the clocks
    sampled meanwhile: the decode figure under sustained load."""
    sp = job.sp

    def call():
        sp.spark_decode_attn(job.q, job.kc, job.v_ev if wl.keep else job.v, job.kt, job.vt, job.cap, 1, wl.G,
                             job.out, job.wsd, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    n = max(10, int(seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3)))
    sampler = ClockSampler(job.dev.index)
    sampler.start()
    time.sleep(0.2)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n):
            call()
        e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if sp.spark_device_status(job.wsd) != 0:
        raise RuntimeError("device status after the sustained decode calls")
    us = e0.elapsed_time(e1) / n * 1e3
    gbs = nbytes / (us / 1e6) / 1e9
    return {"calls": n, "us_per_call": us, "gbs": gbs, "frac_8tbs": gbs / NOMINAL_HBM_GBS,
            f"frac_{peak_kind}": gbs / peak, "clocks": clocks,
            "timing": "CUDA events around n back-to-back spark_decode_attn calls on the launching stream"}


def run_variants(job, wl, stream, peak, peak_kind, iters=5):
    """Method variants on the same prompt, timed outside the step with CUDA
    events on the launching stream: SparK-g grouped pruning with the pages'
    g = 4 rates (0.25, 0.5, 0.75, 1.0), the ThinK structured comparator at the
    same T (prune + decode), SparK-p at p = 0.99 with the full 128-slot
    capacity (prune + decode), and value-channel pruning at lambda_v = 0.5
    with decode over the pruned key and value caches (bf16)."""
    sp = job.sp
    S = job.S_kept
    k = job.k_ev if wl.keep else job.k
    v = job.v_ev if wl.keep else job.v
    es = 2 if wl.dtype == "bf16" else 4

    def timed(f):
        with torch.cuda.stream(stream):
            for _ in range(2):
                f()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(iters):
                f()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters * 1e3

    out = {}
    rates = [0.25, 0.5, 0.75, 1.0]
    Tg = sp.spark_group_budget(wl.D, rates)
    kg = sp.KCache.empty(wl.rows, wl.Hkv, S, wl.D, sum(Tg), wl.torch_dtype, device=job.dev)
    us = timed(lambda: sp.spark_prune_grouped(k, job.q_obs, wl.G, wl.W, Tg, kg, job.wsp, stream))
    nbytes = wl.BH * S * (wl.D * es + 16 + sum(Tg) * es)
    gbs = nbytes / (us / 1e6) / 1e9
    out["spark_g"] = {"rates": rates, "group_T": Tg, "T": sum(Tg), "us_per_call": us, "gbs": gbs,
                      f"frac_{peak_kind}": gbs / peak, "bytes_per_call": nbytes,
                      "timing": "CUDA events around spark_prune_grouped on its stream, outside the step"}
    del kg
    # ThinK comparator at the same T: structured prune, then the same decode
    kt_ = sp.KCache.empty(wl.rows, wl.Hkv, S, wl.D, job.T, wl.torch_dtype, device=job.dev)
    wst = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_THINK, wl.rows, wl.Hkv, wl.G, S, wl.D, job.T, 0),
                       job.dev)
    us_tp = timed(lambda: sp.spark_prune_think(k, job.q_obs, wl.G, wl.W, kt_, wst, stream))
    wsd_t = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_DECODE, wl.rows, wl.Hkv, wl.G, S, wl.D, job.T, 0),
                         job.dev)
    outt = torch.empty_like(job.out)
    us_td = timed(lambda: sp.spark_decode_attn(job.q, kt_, v, None, None, 0, 0, wl.G, outt, wsd_t, stream=stream))
    nb_t = wl.BH * S * (16 + job.T * es + wl.D * es)
    out["think"] = {"T": job.T, "prune_us": us_tp, "prune_bytes": wl.BH * S * (2 * wl.D * es + 16 + job.T * es),
                    "decode_us": us_td, "decode_gbs": nb_t / (us_td / 1e6) / 1e9,
                    "timing": "CUDA events on the stream, outside the step; no tail"}
    del kt_, wst, wsd_t
    # SparK-p at the pages' p = 0.99, full capacity (no cut): prune + decode
    Tcap = wl.D
    kp_ = sp.KCache.empty_topp(wl.rows, wl.Hkv, S, wl.D, Tcap, wl.torch_dtype, device=job.dev)
    wsp_p = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_TOPP, wl.rows, wl.Hkv, wl.G, S, wl.D, Tcap, 0),
                         job.dev)
    us_pp = timed(lambda: sp.spark_prune_topp(k, job.q_obs, wl.G, wl.W, 0.99, kp_, wsp_p, stream))
    n_pruned = float(kp_.stats.reshape(-1, 4)[:, 0].sum().item())
    mean_kept = wl.D - n_pruned / max(wl.BH * S, 1)
    wsd_p = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_DECODE, wl.rows, wl.Hkv, wl.G, S, wl.D, Tcap, 0),
                         job.dev)
    outp = torch.empty_like(job.out)
    us_pd = timed(lambda: sp.spark_decode_attn_topp(job.q, kp_, v, None, None, 0, 0, wl.G, outp, wsd_p,
                                                    stream=stream))
    if sp.spark_device_status(wsd_p) != 0:
        raise RuntimeError("device status after the SparK-p decode")
    # the compact value stream: each 32-token group holds its longest kept set
    used = sp.spark_topp_vals_used(kp_, stream)
    ng = (S + 31) // 32
    nb_pp = wl.BH * S * (2 * wl.D * es + 16) + used + (wl.BH * ng + 1) * 4  # K read twice
    nb_pd = wl.BH * S * (16 + wl.D * es) + used + (wl.BH * ng + 1) * 4
    out["spark_p"] = {"p": 0.99, "Tcap": Tcap, "mean_kept": mean_kept, "mean_prune_rate": 1 - mean_kept / wl.D,
                      "vals_bytes": used, "vals_bytes_per_token_head": used / max(wl.BH * S, 1),
                      "prune_us": us_pp, "prune_bytes": nb_pp, "prune_gbs": nb_pp / (us_pp / 1e6) / 1e9,
                      "decode_us": us_pd, "decode_bytes": nb_pd, "decode_gbs": nb_pd / (us_pd / 1e6) / 1e9,
                      "timing": "CUDA events on the stream, outside the step; no tail"}
    del kp_, wsp_p, wsd_p
    out["decode_loop"] = run_decode_loop(sp, job.dev)
    if wl.dtype == "bf16":
        Tv = sp.spark_lambda_to_T(0.5, wl.D)
        vc = sp.KCache.empty(wl.rows, wl.Hkv, S, wl.D, Tv, wl.torch_dtype, device=job.dev)
        us_p = timed(lambda: sp.spark_prune_values(v, vc, job.wsp, stream))
        wkv = sp.workspace(sp.spark_workspace_bytes_kv(wl.rows, wl.Hkv, wl.G, S, wl.D, job.T, Tv, 0), job.dev)
        outb = torch.empty_like(job.out)
        us_d = timed(lambda: sp.spark_decode_attn_kv(job.q, job.kc, vc, None, None, 0, 0, wl.G, outb, wkv,
                                                     stream))
        if sp.spark_device_status(wkv) != 0:
            raise RuntimeError("device status after the value-pruned decode")
        nb = wl.BH * S * (16 + job.T * es + 16 + Tv * es)
        out["spark_v"] = {"lambda_k": wl.lam, "lambda_v": 0.5, "T": job.T, "Tv": Tv,
                          "prune_values_us": us_p, "decode_us": us_d, "decode_bytes": nb,
                          "decode_gbs": nb / (us_d / 1e6) / 1e9,
                          "decode_token_heads_per_s": wl.BH * S / (us_d / 1e6),
                          "timing": "CUDA events on the stream, outside the step; no tail"}
    return out


def run_decode_loop(sp, dev, steps=64):
    """The decode phase of the single-layer Llama-3.1-8B shape (B=1, 8 kv
    heads x 4, S=32768, lambda=0.5, bf16): 64 steps, each appending the new
    key/value to the dense tail and decoding.  One step moves ~105 MB, a few
    microseconds of HBM time, so launches matter: the same 64 steps are timed
    as individual calls and as one replay of a CUDA graph that captured them."""
    wl = WORKLOADS["llama1l"]
    T = sp.spark_lambda_to_T(wl.lam, wl.D)
    pre = make_prefill(wl, dev)
    R, H, S, D, G = wl.rows, wl.Hkv, wl.S, wl.D, wl.G
    kc = sp.KCache.empty(R, H, S, D, T, wl.torch_dtype, device=dev)
    wsp = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_PRUNE, R, H, G, S, D, T, 0), dev)
    sp.spark_prune(pre["k"], pre["q_obs"], G, wl.W, kc, wsp)
    cap = steps
    kt = torch.zeros((R, H, cap, D), dtype=wl.torch_dtype, device=dev)
    vt = torch.zeros_like(kt)
    ws = sp.workspace(sp.spark_workspace_bytes(sp.SPARK_OP_DECODE, R, H, G, S, D, T, cap), dev)
    stp = [make_decode_step(wl, i, dev) for i in range(steps)]
    out = torch.empty((R, wl.Hq, D), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()

    def loop():
        for i in range(steps):
            sp.spark_tail_append(stp[i]["k_new"], stp[i]["v_new"], kt, vt, R, H, D, cap, i, stream)
            sp.spark_decode_attn(stp[i]["q"], kc, pre["v"], kt, vt, cap, i + 1, G, out, ws, stream=stream)

    def timed(f, reps=5):
        with torch.cuda.stream(stream):
            f()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                f()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps / steps * 1e3

    us_eager = timed(loop)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            loop()
    torch.cuda.synchronize()
    us_graph = timed(g.replay)
    if sp.spark_device_status(ws) != 0:
        raise RuntimeError("device status after the decode loop")
    del g
    es = 2
    nb = wl.BH * S * (16 + T * es + D * es) + wl.BH * (steps // 2) * 2 * D * es  # cache + mean tail
    return {"workload": "llama1l: B=1 L=1 Hkv=8 G=4 S=32768 lambda=0.5 (T=64) bf16, 64 decode steps",
            "us_per_step_eager": us_eager, "us_per_step_graph": us_graph,
            "launches_per_step": 3, "bytes_per_step": nb, "gbs_graph": nb / (us_graph / 1e6) / 1e9,
            "timing": "CUDA events around 5 repetitions of the 64 steps on one stream; tail append + decode "
                      "+ combine per step"}


def run_sweep(args):
    """Every configuration of the workload table on one GPU: prune and one
    decode step (dense tail of one token) timed with CUDA events on the
    launching stream (inputs larger than L2 except `tiny`), each against the
    HBM roofline on its algorithmic bytes.  One JSON object per line."""
    import channel_pruned_decode_b200 as sp
    peak, peak_kind = _peaks()
    dev = "cuda"
    if not args.sweep_workloads:
        # one process per configuration: a configuration timed after another
        # one in the same process can inherit a slow device state (the long
        # prune after the single-layer one: 8.7 ms instead of 4.8)
        for name in ("tiny", "llama1l", "lsweep_0.3", "lsweep_0.5", "lsweep_0.8", "long", "evict"):
            r = subprocess.run([sys.executable, os.path.abspath(__file__), "--sweep", "--sweep-workloads", name],
                               capture_output=True, text=True)
            sys.stdout.write(r.stdout)
            sys.stdout.flush()
            if r.returncode != 0:
                sys.stderr.write(r.stderr)
                raise SystemExit(r.returncode)
        return
    names = args.sweep_workloads.split(",")
    for name in names:
        wl = WORKLOADS[name]
        T = sp.spark_lambda_to_T(wl.lam, wl.D)
        job = Job(wl, dev)
        stream = torch.cuda.Stream()
        k, v = job.k, job.v
        rec = {"workload": _workload_desc(wl, T).split(";")[0], "T": T}

        def timed(f, reps):
            # warm up for at least 0.2 s of device time (and 3 calls): the
            # first calls on freshly allocated buffers run up to 2x slower
            with torch.cuda.stream(stream):
                t_end, n = time.perf_counter() + 0.2, 0
                while n < 3 or time.perf_counter() < t_end:
                    f()
                    n += 1
                    if n % 8 == 0:
                        torch.cuda.synchronize()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    f()
                e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / reps * 1e3

        reps = 5 if name == "long" else 20
        if wl.keep:
            rec["snapkv_us"] = timed(lambda: sp.spark_snapkv_evict(
                job.k, job.v, job.q_obs, wl.G, wl.W, wl.keep, wl.pool, job.k_ev, job.v_ev, job.idx, job.wse,
                stream), reps)
            k, v = job.k_ev, job.v_ev
            sp.spark_snapkv_evict(job.k, job.v, job.q_obs, wl.G, wl.W, wl.keep, wl.pool, job.k_ev, job.v_ev,
                                  job.idx, job.wse, stream)
        S = job.S_kept
        es = 2 if wl.dtype == "bf16" else 4
        us_p = timed(lambda: sp.spark_prune(k, job.q_obs, wl.G, wl.W, job.kc, job.wsp, stream), reps)
        sp.spark_tail_append(job.k_new, job.v_new, job.kt, job.vt, wl.rows, wl.Hkv, wl.D, job.cap, 0, stream)
        us_d = timed(lambda: sp.spark_decode_attn(job.q, job.kc, v, job.kt, job.vt, job.cap, 1, wl.G, job.out,
                                                  job.wsd, stream=stream), reps)
        if sp.spark_device_status(job.wsd) != 0:
            raise RuntimeError(f"device status after decode ({name})")
        bp = wl.BH * S * (wl.D * es + 16 + T * es)
        bd = wl.BH * S * (16 + T * es + wl.D * es) + wl.BH * 2 * wl.D * es
        rec.update({"prune_us": us_p, "prune_gbs": bp / (us_p / 1e6) / 1e9,
                    f"prune_frac_{peak_kind}": bp / (us_p / 1e6) / 1e9 / peak,
                    "decode_us": us_d, "decode_gbs": bd / (us_d / 1e6) / 1e9,
                    f"decode_frac_{peak_kind}": bd / (us_d / 1e6) / 1e9 / peak,
                    "decode_token_heads_per_s": wl.BH * (S + 1) / (us_d / 1e6),
                    "l2": "inputs exceed the 126 MB L2" if bd > 126e6 else "inputs fit in L2 (parity-size case)"})
        print(json.dumps(rec), flush=True)
        del job
        torch.cuda.empty_cache()


def run_e2e(job, wl, steps, dist_on, world):
    """Same metric through the public API with pinned HOST inputs: every step
    copies K, V, window queries and the decode query/new key/value to the
    device, runs the step and reads the output back."""
    import psutil
    need = sum(t.numel() * t.element_size() for t in (job.k, job.v, job.q_obs, job.q, job.k_new, job.v_new))
    if psutil.virtual_memory().available < 2.5 * need:
        return {"value": None, "unit": UNIT, "skipped": f"host RAM < 2.5 x {need / 1e9:.1f} GB"}
    hk = torch.empty(job.k.shape, dtype=job.k.dtype, pin_memory=True)
    hv = torch.empty(job.v.shape, dtype=job.v.dtype, pin_memory=True)
    hk.copy_(job.k)
    hv.copy_(job.v)
    small = [(torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t), t)
             for t in (job.q_obs, job.q, job.k_new, job.v_new)]
    hout = torch.empty(job.out.shape, dtype=job.out.dtype, pin_memory=True)
    stream = torch.cuda.Stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def one():
        job.k.copy_(hk, non_blocking=True)
        job.v.copy_(hv, non_blocking=True)
        for h, d in small:
            d.copy_(h, non_blocking=True)
        job.step(stream)
        hout.copy_(job.out, non_blocking=True)

    with torch.cuda.stream(stream):
        one()
    torch.cuda.synchronize()
    _barrier(dist_on)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            one()
        end.record(stream)
    torch.cuda.synchronize()
    ms = _max_over_ranks(start.elapsed_time(end), dist_on) / steps
    h2d = need
    d2h = hout.numel() * hout.element_size()
    return {"value": world * wl.BH * (wl.S_kept + 1) / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps}


# -------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import concurrent.futures as cf

    import oracle
    lib = oracle.load()
    wl = WORKLOADS[args.workload]
    T = oracle.lambda_to_T(wl.lam, wl.D, lib=lib)
    cores = os.cpu_count() or 1
    S, D, G = wl.S, wl.D, wl.G
    # one step = `cores` (kv head) units of the first S_s prompt tokens: prune +
    # one decode step each; bounded so that K + W steps take a few minutes
    S_s = min(S, 16384)
    wl1 = scaled(wl, L=1, B=1, S=S_s)
    pre = make_prefill(wl1, "cpu")
    stp = make_decode_step(wl1, 0, "cpu")
    units = []
    for u in range(cores):
        h = u % wl.Hkv
        units.append((pre["k"][0, h:h + 1].float().numpy(), pre["v"][0, h:h + 1].float().numpy(),
                      pre["q_obs"][0, h * G:(h + 1) * G].float().numpy(),
                      stp["q"][0, h * G:(h + 1) * G].float().numpy()))

    def one(d):
        kk, vv, qq, q1 = d
        qn = oracle.qnorm(qq, G, lib=lib)
        m, vals, st = oracle.prune(kk, qn, T, lib=lib)
        return oracle.decode(q1, m, vals, qn, st, vv, G=G, lib=lib)

    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        for _ in range(args.warmup):
            list(ex.map(one, units))
        t0 = time.perf_counter()
        for _ in range(args.steps):
            list(ex.map(one, units))
        dt = time.perf_counter() - t0
    value = args.steps * len(units) * (S_s + 1) / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": _workload_desc(wl, T)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {len(units)} kv-head units of the first {S_s} of "
                                   f"S={S} prompt tokens, prune + 1 decode step (threads over units)",
                         "cpu_model": _cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="spark", choices=["spark", "reference"])
    ap.add_argument("--workload", default="long", choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (small profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip the SparK-g variant timing")
    ap.add_argument("--sweep", action="store_true",
                    help="time prune and decode on every workload (one JSON line each) instead of the step")
    ap.add_argument("--sweep-workloads", default="", help="comma-separated subset for --sweep")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
