"""Benchmark of the SpecOPD branch-scoring hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  specopd_tree_build  (parent map, semantic positions, score rows)
  specopd_tree_attn   (branch RoPE + tensor-core tree attention, one layer)
  specopd_e2e_tv      (overlaps, prefix products, loss, d loss / d draft logits)
on the 8B-shaped workload (T=4096, B=64 anchors over the response half, W=8,
32 q / 8 kv heads, head_dim 128, bf16; vocab 151,936, N = 512 positions).
The trunk K cache comes from specopd_trunk_prefill (causal attention of the
trunk with the K cache written rotated), run once before timing: the trunk is
prefilled once and shared by all of its branches.  Its time is reported
beside the step (`prefill`), not inside it.

Metric: scored branch rows per second, R = B(W-1) rows per step and per GPU.
Multi-GPU (torchrun): every rank scores its own batch of branches (weak
scaling); the only exchange is the distributed normalisation of the loss
(one all-reduce of the prefix-product sum; the gradient already uses the
global position count), as the method prescribes for ranks with different
numbers of scored positions.

--impl reference times the fp64 CPU oracle (the only reference this method
has: no implementation was released) on a bounded sample of the same
workload, on this machine's host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "8b"  # default; --workload selects another of the synthetic configs
WORKLOAD_NAMES = {
    "tiny": "tiny fp32: T=256, B=4, W=4, 4q/1kv heads, head_dim 64, vocab 1024, N=16 positions",
    "8b": "8B-shaped single layer: T=4096, B=64 anchors, W=8, 32q/8kv heads, head_dim 128, "
          "vocab 151936, N=512 positions",
    "long": "long trunk: T=32768, B=256 anchors, W=16, 40q/8kv heads, head_dim 128, vocab 151936, "
            "N=4096 positions",
    "packed": "packed batch: 8 sequences of 2048-16384 tokens, B=128 anchors each, W=16, "
              "64q/8kv heads, head_dim 128, vocab 248320, N=16384 positions",
}
METRIC = "scored branch rows/s (tree-attn + E2E-TV); % of bf16 TC peak and HBM roofline"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "src": "fallback"}


def attention_flops(cfg, anchors):
    """Algorithmic FLOPs: sum over rows and q heads of 4*D*(a_b + 1 + i)
    (QK^T and PV over the visible keys only)."""
    W = cfg.W
    keys = 0
    for a in anchors:
        keys += sum(int(a) + 1 + i for i in range(1, W))
    return 4.0 * cfg.D * cfg.Hq * keys


def prefill_flops(cfg, cu):
    """Algorithmic FLOPs of the trunk prefill: every trunk row t (position p
    in its sequence) and q head scores and mixes p + 1 keys, 4*D each."""
    keys = 0
    for s in range(len(cu) - 1):
        T = cu[s + 1] - cu[s]
        keys += T * (T + 1) // 2
    return 4.0 * cfg.D * cfg.Hq * keys


def _clock_sampler(path):
    cmd = ["nvidia-smi", "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
           "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
           "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
           "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "100"]
    try:
        f = open(path, "w")
        return subprocess.Popen(cmd, stdout=f, stderr=subprocess.DEVNULL), f
    except Exception:
        return None, None


def _clock_summary(path, dev_index):
    sm, smax, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    try:
        for line in open(path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9 or p[0] != str(dev_index):
                continue
            try:
                sm.append(float(p[1]))
                smax = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
    except FileNotFoundError:
        pass
    return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
            "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ device problem

class Problem:
    """Device-resident inputs and outputs of one step of a named workload."""

    def __init__(self, torch, api, dev, seed_offset=0, workload=WORKLOAD):
        self.torch, self.api, self.dev = torch, api, dev
        acfg = synth.attn_config(workload)
        tcfg = synth.tv_config(workload)
        self.acfg, self.tcfg = acfg, tcfg
        inp = synth.attention_inputs(acfg)
        self.inp = inp
        adt = torch.bfloat16 if acfg.dtype == "bf16" else torch.float32
        ldt = torch.bfloat16 if tcfg.dtype == "bf16" else torch.float32
        bf = ldt
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev).to(adt)  # noqa
        self.cu_host = [int(c) for c in inp.cu_trunk]
        self.cu_dev = torch.tensor(inp.cu_trunk, device=dev)
        self.anchors = torch.tensor(inp.anchors, device=dev)
        self.q_br, self.k_br, self.v_br = t(inp.q_br), t(inp.k_br), t(inp.v_br)
        self.k_tr, self.v_tr = t(inp.k_tr), t(inp.v_tr)
        S, B, W = acfg.S, acfg.B, acfg.W
        self.R = S * B * (W - 1)
        self.N = S * B * W
        self.T_tot = inp.T_tot
        i32 = torch.int32
        self.parent = torch.empty(self.T_tot + self.R, dtype=i32, device=dev)
        self.sem_pos = torch.empty(self.T_tot + self.R, dtype=i32, device=dev)
        self.score_row = torch.empty(self.N, dtype=i32, device=dev)
        api.specopd_tree_build(self.cu_host, self.anchors, B, W, self.parent, self.sem_pos,
                               self.score_row)
        self.desc = api.attn_desc(S, B, W, acfg.Hq, acfg.Hkv, acfg.D, acfg.dtype, acfg.rope_base)
        # Trunk prefill: trunk queries (seeded, N(0,1)), the raw trunk keys
        # kept for timing it again, the K cache rotated in place by the call.
        gq = torch.Generator(device=dev)
        gq.manual_seed(4321 + seed_offset)
        self.q_tr = torch.randn((self.T_tot, acfg.Hq, acfg.D), generator=gq, device=dev).to(adt)
        self.k_raw = self.k_tr.clone()
        self.out_tr = torch.empty_like(self.q_tr)
        self.pf_ws = torch.empty(max(api.specopd_trunk_prefill_workspace_size(self.desc,
                                                                              self.cu_host), 256),
                                 dtype=torch.uint8, device=dev)
        api.specopd_trunk_prefill(self.desc, self.q_tr, self.k_tr, self.v_tr, self.cu_dev,
                                  self.cu_host, out=self.out_tr, workspace=self.pf_ws)
        self.pf_flops = prefill_flops(acfg, self.cu_host)
        ws = api.specopd_tree_attn_workspace_size(self.desc, self.cu_host)
        self.attn_ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(self.q_br)
        # logits: target rows in packed node order [T_tot + R, V], read through
        # the score-row map; draft logits [N, V].  Rows are generated on the
        # device with the per-row recipe's distribution (seeded torch RNG), the
        # oracle-checked rows come from synth on the host (tests).
        V = tcfg.V
        self.V = V
        g = torch.Generator(device=dev)
        g.manual_seed(1234 + seed_offset)
        rows_t = self.T_tot + self.R
        self.rows_t = rows_t
        self.z_t = torch.zeros((rows_t, V), dtype=bf, device=dev)
        self.z_d = torch.empty((self.N, V), dtype=bf, device=dev)
        sr = self.score_row.long()
        for n0 in range(0, self.N, 2048):  # row chunks bound the fp32 temporaries
            n1 = min(self.N, n0 + 2048)
            zt = torch.randn((n1 - n0, V), generator=g, device=dev) * tcfg.sigma_t
            k = torch.randint(1, 4, (n1 - n0,), generator=g, device=dev)
            ids = torch.randint(0, V, (n1 - n0, 3), generator=g, device=dev)
            bump = (torch.arange(3, device=dev)[None, :] < k[:, None]).float() * tcfg.bump
            zt.scatter_add_(1, ids, bump)
            zd = zt + torch.randn((n1 - n0, V), generator=g, device=dev) * tcfg.sigma_d
            self.z_t[sr[n0:n1]] = zt.to(bf)
            self.z_d[n0:n1] = zd.to(bf)
            del zt, zd
        torch.cuda.synchronize()
        self.tdesc = api.tv_desc(S * B, W, V, rows_t, tcfg.dtype, "f32", True,
                                 norm_count=self.N)
        self.tv_ws = torch.empty(api.specopd_e2e_tv_workspace_size(self.tdesc), dtype=torch.uint8,
                                 device=dev)
        f32 = torch.float32
        self.a = torch.empty(self.N, dtype=f32, device=dev)
        self.prefix = torch.empty(self.N, dtype=f32, device=dev)
        self.loss = torch.empty(1, dtype=f32, device=dev)
        self.numer = torch.empty(1, dtype=torch.float64, device=dev)
        self.grad = torch.empty((self.N, V), dtype=f32, device=dev)
        self.flops = attention_flops(acfg, inp.anchors)
        es = 2 if tcfg.dtype == "bf16" else 4
        self.tv_bytes = float(self.N) * V * (2 * es + 4)

    def step(self, ev=None):
        api, acfg = self.api, self.acfg
        api.specopd_tree_build(self.cu_host, self.anchors, acfg.B, acfg.W, self.parent,
                               self.sem_pos, self.score_row)
        if ev is not None:
            ev[0].record()
        api.specopd_tree_attn(self.desc, self.q_br, self.k_br, self.v_br, self.k_tr, self.v_tr,
                              self.cu_dev, self.cu_host, self.anchors, self.sem_pos, out=self.out,
                              workspace=self.attn_ws)
        if ev is not None:
            ev[1].record()
        api.specopd_e2e_tv(self.tdesc, self.z_t, self.score_row, self.z_d, a=self.a,
                           prefix=self.prefix, loss=self.loss, numer=self.numer, grad=self.grad,
                           workspace=self.tv_ws)
        if ev is not None:
            ev[2].record()


    def time_prefill(self, reps=5):
        """Device time (ms) of one specopd_trunk_prefill, on a fresh copy of
        the raw trunk keys each time (the call rotates them in place; the
        copy is outside the timed region)."""
        torch = self.torch
        k = torch.empty_like(self.k_raw)
        evs = []
        for i in range(reps + 2):
            k.copy_(self.k_raw)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            self.api.specopd_trunk_prefill(self.desc, self.q_tr, k, self.v_tr, self.cu_dev,
                                           self.cu_host, out=self.out_tr, workspace=self.pf_ws)
            e1.record()
            if i >= 2:
                evs.append((e0, e1))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / len(evs)


def kernels_per_step(acfg):
    """Library kernels one step launches: tree_build, tree_attn (branch RoPE
    fused for bf16; a separate RoPE launch for the fp32 SIMT path), e2e_tv."""
    return 3 if acfg.dtype == "bf16" else 4


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from tree_attention_specopd_b200 import api
    from tree_attention_specopd_b200 import dist as sdist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    api.load()
    wl = args.workload
    pb = Problem(torch, api, dev, seed_offset=rank, workload=wl)
    # Distributed normalisation: every rank's gradient and loss divide by the
    # GLOBAL position count (gathered once), and the prefix-product sums are
    # all-reduced after each step.
    n_global = sdist.global_count(pb.N, device=dev)
    if world > 1:
        pb.tdesc = api.tv_desc(pb.acfg.S * pb.acfg.B, pb.acfg.W, pb.V, pb.rows_t, pb.tcfg.dtype, "f32",
                               True, norm_count=n_global)
    numer_all = torch.zeros(1, dtype=torch.float64, device=dev)
    loss_all = torch.zeros(1, dtype=torch.float64, device=dev)

    def full_step(ev=None):
        pb.step(ev)
        if world > 1:
            numer_all.copy_(pb.numer)
            loss_all.copy_(sdist.global_loss(numer_all, n_global))

    for _ in range(args.warmup):
        full_step()
    torch.cuda.synchronize()
    st = api.specopd_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after warm-up")

    import tempfile
    clk_path = os.path.join(tempfile.gettempdir(), f"specopd_clocks_rank{rank}.csv")
    sampler, fh = _clock_sampler(clk_path) if rank == 0 else (None, None)
    time.sleep(0.3 if sampler else 0)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    for k in range(args.steps):
        full_step(evs[k])
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    attn_ms = sum(ev[0].elapsed_time(ev[1]) for ev in evs) / args.steps
    tv_ms = sum(ev[1].elapsed_time(ev[2]) for ev in evs) / args.steps
    if sampler:
        sampler.terminate()
        sampler.wait()
        fh.close()
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    loss = float(pb.loss.item())
    st = api.specopd_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after the timed steps")

    # ---- end-to-end through the public API with host buffers (the default
    # workload; the larger ones would copy tens of GB per step)
    e2e = e2e_measure(torch, api, pb, args, dev, world) if wl == WORKLOAD else None
    pf_ms = pb.time_prefill() if rank == 0 else None

    # ---- the other workloads, device-timed in the same run (one GPU)
    extra = None
    lmhead = None
    if world == 1 and wl == WORKLOAD and not args.no_extra_workloads:
        figs = _Figures(pb)
        del pb
        torch.cuda.empty_cache()
        extra = {}
        for other in ("tiny", "long", "packed"):
            extra[other] = measure_workload(torch, api, dev, other, max(3, min(args.steps, 10)),
                                            args.warmup)
            torch.cuda.empty_cache()
        lmhead = measure_lmhead_tv(torch, api, dev)
        pb = figs

    if rank == 0:
        peaks = _peaks()
        ms_step = ms_max / args.steps
        value = pb.R * world / (ms_step / 1e3)
        tv_gbs = pb.tv_bytes / (tv_ms / 1e3) / 1e9
        attn_tflops = pb.flops / (attn_ms / 1e3) / 1e12
        pf_tflops = pb.pf_flops / (pf_ms / 1e3) / 1e12 if pf_ms else None
        clocks = _clock_summary(clk_path, local)
        traffic = _ncu_traffic() if wl == WORKLOAD else None  # counters of the 8B launch
        # DRAM bytes actually moved per launch (ncu) over the live launch time:
        # re-reads that miss L2 count here and not in `achieved`
        dram_gbs = traffic / (tv_ms / 1e3) / 1e9 if traffic else None
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "rows/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": pb.acfg.dtype,
            "data": "synthetic",
            "config": {"workload": WORKLOAD_NAMES[wl],
                       "rows_per_step_per_gpu": pb.R, "positions_per_step_per_gpu": pb.N,
                       "parallelism": f"dp{world} (branch batches per rank)",
                       "l2": (f"inputs larger than L2 ({pb.tv_bytes / 2e9:.2f} GB of logits read "
                              "per step vs 126 MB)") if pb.tv_bytes / 2 > 126e6 else
                             "inputs fit in L2 (small workload; not an HBM measurement)"},
            "supervised_tokens_per_s": pb.N * world / (ms_step / 1e3),
            "roofline": {"bound": "hbm", "kernel": "e2e_tv", "achieved": tv_gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": tv_gbs / peaks["hbm_gbs"], "traffic": traffic,
                         "dram_gbs": dram_gbs,
                         "dram_frac": dram_gbs / peaks["hbm_gbs"] if dram_gbs else None,
                         "algorithmic_bytes_per_launch": pb.tv_bytes, "launch_ms": tv_ms,
                         "peak_src": peaks["src"]},
            "attention_roofline": {"bound": "tensor" if pb.acfg.dtype == "bf16" else "fp32 SIMT",
                                   "kernel": "tree_attn", "achieved": attn_tflops,
                                   "peak": peaks["bf16_tflops"] if pb.acfg.dtype == "bf16" else None,
                                   "unit": "TFLOP/s",
                                   "frac": attn_tflops / peaks["bf16_tflops"]
                                   if pb.acfg.dtype == "bf16" else None,
                                   "algorithmic_flops_per_launch": pb.flops, "launch_ms": attn_ms,
                                   "peak_src": peaks["src"]},
            "prefill": {"kernel": "tree_attn (trunk prefill mode) + K-cache RoPE",
                        "note": "once per trunk, before the timed steps; not part of a step",
                        "launch_ms": pf_ms, "algorithmic_flops_per_call": pb.pf_flops,
                        "achieved": pf_tflops, "unit": "TFLOP/s",
                        "peak": peaks["bf16_tflops"] if pb.acfg.dtype == "bf16" else None,
                        "frac": pf_tflops / peaks["bf16_tflops"]
                        if pf_tflops and pb.acfg.dtype == "bf16" else None},
            "loss": loss,
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": kernels_per_step(pb.acfg) * args.steps,
        }
        if extra is not None:
            line["workloads"] = extra
        if lmhead is not None:
            line["lmhead_tv"] = lmhead
        if e2e is None:
            line["e2e_note"] = "host-buffer end-to-end measured on the default 8B workload only"
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds, workload=wl)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


class _Figures:
    """Per-step constants of a Problem (sizes, algorithmic work), kept after
    its device buffers are released."""

    def __init__(self, pb):
        for k in ("acfg", "tcfg", "R", "N", "flops", "pf_flops", "tv_bytes"):
            setattr(self, k, getattr(pb, k))


def measure_workload(torch, api, dev, workload, steps, warmup):
    """Device-timed step of another workload (CUDA events on the launching
    stream, as for the main line): rows/s and both roofline fractions."""
    pb = Problem(torch, api, dev, workload=workload)
    for _ in range(warmup):
        pb.step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(steps):
        pb.step(evs[k])
    e1.record()
    torch.cuda.synchronize()
    st = api.specopd_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} on the {workload} workload")
    peaks = _peaks()
    ms = e0.elapsed_time(e1) / steps
    attn_ms = sum(ev[0].elapsed_time(ev[1]) for ev in evs) / steps
    tv_ms = sum(ev[1].elapsed_time(ev[2]) for ev in evs) / steps
    pf_ms = pb.time_prefill(3)
    bf = pb.acfg.dtype == "bf16"
    tv_gbs = pb.tv_bytes / (tv_ms / 1e3) / 1e9
    att = pb.flops / (attn_ms / 1e3) / 1e12
    pft = pb.pf_flops / (pf_ms / 1e3) / 1e12
    out = {"workload": WORKLOAD_NAMES[workload], "steps": steps, "warmup": warmup,
           "ms_per_step": ms, "value": pb.R / (ms / 1e3), "unit": "rows/s",
           "supervised_tokens_per_s": pb.N / (ms / 1e3),
           "e2e_tv": {"launch_ms": tv_ms, "achieved_gbs": tv_gbs,
                      "frac": tv_gbs / peaks["hbm_gbs"],
                      "algorithmic_bytes_per_launch": pb.tv_bytes},
           "tree_attn": {"launch_ms": attn_ms, "achieved_tflops": att,
                         "frac": att / peaks["bf16_tflops"] if bf else None,
                         "algorithmic_flops_per_launch": pb.flops},
           "prefill": {"launch_ms": pf_ms, "achieved_tflops": pft,
                       "frac": pft / peaks["bf16_tflops"] if bf else None},
           "peak_src": peaks["src"],
           "l2": "inputs larger than L2" if pb.tv_bytes / 2 > 126e6 else "inputs fit in L2"}
    del pb
    return out


def measure_lmhead_tv(torch, api, dev, nbranch=64, W=8, V=151936, d=4096, reps=5, warmup=2):
    """Device time of specopd_e2e_tv_lmhead (the LM heads fused in front of
    E2E-TV) on the 8B shape with a 4096-wide hidden state: seeded bf16 hidden
    rows and heads made on the device with the synth recipe's distributions,
    CUDA events around `reps` calls after `warmup`.  Executed tensor work
    with the fp32 gradient: passes 0 and 1 form both models' logits (4 GEMMs
    of 2 N V d FLOPs); the gradient is then scaled in place."""
    N = nbranch * W
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    sc = 3.0 / d ** 0.5
    wt = (torch.randn(V, d, device=dev, generator=g) * sc).to(torch.bfloat16)
    wd = (wt.float() + torch.randn(V, d, device=dev, generator=g) * (0.5 * sc)).to(torch.bfloat16)
    ht = torch.randn(N, d, device=dev, generator=g).to(torch.bfloat16)
    hd = (ht.float() + 0.5 * torch.randn(N, d, device=dev, generator=g)).to(torch.bfloat16)
    desc = api.lmhead_tv_desc(nbranch, W, V, d, N, "f32", True)
    ws = torch.empty(api.specopd_e2e_tv_lmhead_workspace_size(desc), dtype=torch.uint8, device=dev)
    out = {"a": torch.empty(N, device=dev), "prefix": torch.empty(N, device=dev),
           "loss": torch.empty(1, device=dev),
           "numer": torch.empty(1, dtype=torch.float64, device=dev),
           "grad": torch.empty((N, V), device=dev)}
    for _ in range(warmup):
        api.specopd_e2e_tv_lmhead(desc, ht, None, wt, hd, wd, workspace=ws, **out)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        api.specopd_e2e_tv_lmhead(desc, ht, None, wt, hd, wd, workspace=ws, **out)
    e1.record()
    torch.cuda.synchronize()
    st = api.specopd_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after specopd_e2e_tv_lmhead")
    ms = e0.elapsed_time(e1) / reps
    flops = 4 * 2.0 * N * V * d
    peaks = _peaks()
    tf = flops / (ms / 1e3) / 1e12
    res = {"call": "specopd_e2e_tv_lmhead", "nbranch": nbranch, "W": W, "V": V, "d_model": d,
           "grad_dtype": "f32", "launch_ms": ms, "executed_flops_per_call": flops,
           "achieved": tf, "unit": "TFLOP/s", "bound": "tensor", "peak": peaks["bf16_tflops"],
           "frac": tf / peaks["bf16_tflops"], "peak_src": peaks["src"],
           "positions_per_s": N / (ms / 1e3),
           "logit_bytes_not_stored": 2 * N * V * 2}
    del wt, wd, ht, hd, ws, out
    torch.cuda.empty_cache()
    return res


TV_SOURCES = (
    "tree_attention_specopd_b200/csrc/e2e_tv.cu",
    "tree_attention_specopd_b200/csrc/e2e_tv_row.cuh",
    "tree_attention_specopd_b200/csrc/common.cuh",
)


def strip_c_comments(src):
    """C/C++ source without its comments, whitespace runs collapsed to one
    space (string and character literals kept as they are)."""
    out, i, n, quote = [], 0, len(src), None
    while i < n:
        c = src[i]
        if quote is None:
            if src.startswith("//", i):
                j = src.find("\n", i)
                i = n if j < 0 else j
                continue
            if src.startswith("/*", i):
                j = src.find("*/", i + 2)
                i = n if j < 0 else j + 2
                out.append(" ")
                continue
            if c in "\"'":
                quote = c
        elif c == "\\" and i + 1 < n:
            out.append(src[i:i + 2])
            i += 2
            continue
        elif c == quote:
            quote = None
        out.append(c)
        i += 1
    return " ".join("".join(out).split())


def source_digest(texts):
    """SHA-256 over sources with comments and layout removed: what the
    compiler sees of them, so an edit of a comment keeps the digest."""
    import hashlib
    h = hashlib.sha256()
    for t in texts:
        h.update(strip_c_comments(t).encode())
        h.update(b"\0")
    return h.hexdigest()


def tv_source_sha256():
    """Digest of the E2E-TV kernel sources (the counters below belong to it)."""
    texts = []
    for rel in TV_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            texts.append(f.read())
    return source_digest(texts)


def _ncu_traffic():
    """DRAM bytes per e2e_tv launch of the 8B-shaped workload from the
    committed ncu summary, or None when it is absent or was taken on other
    kernel sources."""
    path = os.path.join(ROOT, "profiles", "e2e_tv_8b_traffic.json")
    try:
        rec = json.load(open(path))
        if rec.get("source_sha256") != tv_source_sha256():
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


def e2e_measure(torch, api, pb, args, dev, world):
    """Same metric through the public API, host buffers.  Every step uploads
    the step's inputs from pinned host memory -- branch q/k/v, anchors, the
    draft logits, and the target rows straight into the packed table the
    kernel reads through the score-row map (the W-1 branch rows of every
    branch as one block, each anchor's trunk row on its own) -- runs the
    step, and reads the step's results back: the fp32 gradient of the draft
    logits, the attention output and the loss.

    Steps are pipelined over two sets of device buffers, as a training loop
    would run them: while step i computes on one set, the copy streams
    upload step i+1's inputs into the other and read step i-1's results
    out of it.  Events order the three streams: a set's inputs are
    overwritten only after the step that read them finished, and its outputs
    only after they were copied out.  The timed region runs from before the
    first upload to after the last read-back."""
    import torch.distributed as dist
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    T, R = pb.T_tot, pb.R
    sr = pb.score_row.cpu().numpy()
    W = pb.acfg.W
    anchor_rows = [int(sr[b * W]) for b in range(pb.N // W)]  # position (b, 1): a trunk row
    h = {"q": pin(pb.q_br), "k": pin(pb.k_br), "v": pin(pb.v_br), "anc": pin(pb.anchors),
         "zt_br": pin(pb.z_t[T: T + R]), "zt_anc": pin(pb.z_t[anchor_rows]), "zd": pin(pb.z_d)}
    names = ("q_br", "k_br", "v_br", "anchors", "z_t", "z_d", "out", "grad", "loss")
    sets = [{n: getattr(pb, n) for n in names},
            {n: torch.empty_like(getattr(pb, n)) for n in names}]
    outs = [{"grad": torch.empty(pb.grad.shape, dtype=pb.grad.dtype).pin_memory(),
             "out": torch.empty(pb.out.shape, dtype=pb.out.dtype).pin_memory(),
             "loss": torch.empty(1, dtype=torch.float32).pin_memory()} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = sum(t.numel() * t.element_size() for t in outs[0].values())
    # The step runs on a stream of its own: on the legacy default stream its
    # work would serialise with the copy streams' (implicit synchronisation).
    comp, up, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    done = [None, None]     # compute of the set's last step finished
    copied = [None, None]   # read-back of the set's last results finished

    def one(i):
        s = i & 1
        b = sets[s]
        with torch.cuda.stream(up):
            if done[s] is not None:
                up.wait_event(done[s])
            b["q_br"].copy_(h["q"], non_blocking=True)
            b["k_br"].copy_(h["k"], non_blocking=True)
            b["v_br"].copy_(h["v"], non_blocking=True)
            b["anchors"].copy_(h["anc"], non_blocking=True)
            b["z_t"][T: T + R].copy_(h["zt_br"], non_blocking=True)
            for j, row in enumerate(anchor_rows):
                b["z_t"][row].copy_(h["zt_anc"][j], non_blocking=True)
            b["z_d"].copy_(h["zd"], non_blocking=True)
            ready = ev()
            ready.record(up)
        comp.wait_event(ready)
        if copied[s] is not None:
            comp.wait_event(copied[s])
        for n in names:
            setattr(pb, n, b[n])
        with torch.cuda.stream(comp):
            pb.step()
        d = ev()
        d.record(comp)
        done[s] = d
        with torch.cuda.stream(down):
            down.wait_event(d)
            outs[s]["grad"].copy_(b["grad"], non_blocking=True)
            outs[s]["out"].copy_(b["out"], non_blocking=True)
            outs[s]["loss"].copy_(b["loss"], non_blocking=True)
            c = ev()
            c.record(down)
        copied[s] = c

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    steps = max(2, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(comp)
    up.wait_event(e0)
    for i in range(steps):
        one(i)
    comp.wait_event(copied[0])
    comp.wait_event(copied[1])
    e1.record(comp)
    torch.cuda.synchronize()
    for n in names:  # the bench's own buffers again
        setattr(pb, n, sets[0][n])
    ms = e0.elapsed_time(e1) / steps
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    last = outs[(steps - 1) & 1]
    ok = bool(torch.isfinite(last["grad"]).all()) and \
        abs(float(last["loss"].item()) - float(pb.loss.item())) == 0
    return {"value": pb.R * world / (ms / 1e3), "unit": "rows/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "pipelined": "two buffer sets; uploads, step and read-back on three non-default streams",
            "results_read_back": ["grad_draft (fp32)", "attention out", "loss"],
            "read_back_finite": ok}


# ------------------------------------------------------------------ CPU oracle

def cpu_baseline(seconds=15.0, nbranch=None, workload=WORKLOAD):
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    whole branches (their W-1 attention rows and W TV positions), timed on
    the host cores; reported in the bench's unit (scored rows/s)."""
    from oracle import attention as oatt
    from oracle import tv as otv
    acfg = synth.attn_config(workload)
    tcfg = synth.tv_config(workload)
    inp = synth.attention_inputs(acfg)
    rows = 0
    t0 = time.perf_counter()
    b = 0
    while True:
        oatt.branch_attention_unrolled(inp.q_br, inp.k_br, inp.v_br, inp.k_tr, inp.v_tr,
                                       inp.cu_trunk, inp.anchors, acfg.B, acfg.W,
                                       acfg.rope_base, branches=[b])
        zt, zd = synth.logits(tcfg, positions=range(b * acfg.W, (b + 1) * acfg.W))
        otv.e2e_tv(zt, None, zd, 1, acfg.W, norm_count=tcfg.nbranch * acfg.W)
        rows += acfg.W - 1
        b += 1
        el = time.perf_counter() - t0
        if (nbranch is not None and b >= nbranch) or (nbranch is None and el >= seconds) \
                or b >= acfg.B:
            break
    el = time.perf_counter() - t0
    try:
        import threadpoolctl
        threads = max(int(x.get("num_threads", 1)) for x in threadpoolctl.threadpool_info()) \
            if threadpoolctl.threadpool_info() else 1
    except Exception:
        threads = os.cpu_count()
    return {"value": rows / el, "unit": "rows/s", "cores": threads, "kind": "oracle",
            "sample": f"{b} of {acfg.S * acfg.B} branches of the {workload} workload "
                      f"({rows} rows, {b * acfg.W} TV positions) in {el:.1f} s; "
                      f"host has {os.cpu_count()} cores"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per = []
    wl = args.workload
    W = synth.attn_config(wl).W
    for _ in range(args.warmup):
        cpu_baseline(nbranch=1, workload=wl)
    t0 = time.perf_counter()
    rows = 0
    for _ in range(args.steps):
        r = cpu_baseline(nbranch=1, workload=wl)
        rows += W - 1
        per.append(r)
    el = time.perf_counter() - t0
    value = rows / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_NAMES[wl] + " (one branch of it per step)"},
            "cpu_baseline": {"value": value, "unit": "rows/s", "kind": "oracle",
                             "cores": per[-1]["cores"] if per else os.cpu_count(),
                             "sample": f"1 branch ({W - 1} attention rows, {W} TV positions) "
                                       "per step"},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the device-timed secondary workloads of the default run")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(WORKLOAD_NAMES),
                    help="synthetic configuration (default: the 8B-shaped one)")
    ap.add_argument("--lmhead-only", action="store_true",
                    help="time only specopd_e2e_tv_lmhead (the LM heads fused in front of "
                         "E2E-TV) and print its JSON object")
    ap.add_argument("--lmhead-vocab", type=int, default=151936,
                    help="vocabulary of the --lmhead-only run (smaller for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.lmhead_only:
        import torch
        from tree_attention_specopd_b200 import api
        res = measure_lmhead_tv(torch, api, torch.device("cuda", 0), V=args.lmhead_vocab,
                                reps=args.steps, warmup=args.warmup)
        print(json.dumps(res), flush=True)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
