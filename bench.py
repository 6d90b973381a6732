"""Benchmark of the block-sparse causal prefill path (pool -> search -> sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--tau T] [--no-e2e] [--no-cpu-baseline]

One step = one pass of the whole path over the resident synthetic inputs of the workload
(default: Llama-3-8B attention shape, 32 q / 8 kv heads, d = 128, L = 131072, B = 128,
tau = 0.05). The metric is the sparse-prefill time and its effective TFLOP/s (FLOPs of the kept
blocks: 4*B^2*d per off-diagonal block, 2*B^2*d per diagonal block, per head); dense-equivalent
FLOPs, the own-dense time and the speedup over it are reported alongside.

Multi-GPU (torchrun): the path does not shard, so each rank runs an independent replica of the
workload (weak scaling); times are the max over ranks.

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "llama3-8b-L131072"
METRIC = "sparse prefill ms & effective TFLOPS at 128K; % bf16 TC peak; x vs own dense"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16_tflops": float(m["bf16_tflops"]),
                "bf16_tflops_sustained": float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu record, if it was taken on these exact sources."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for rel in rec["sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if rec["kernel"] != kernel or rec["workload"] != workload or h.hexdigest() != rec["sources_sha256"]:
            return None
        return rec["dram_bytes_read"] + rec["dram_bytes_write"]
    except Exception:
        return None


def kept_flops(counts: np.ndarray, cu: np.ndarray, B: int, d: int) -> tuple[float, float]:
    """(effective FLOPs over kept blocks, dense-equivalent causal FLOPs).

    Per head and query block i with n_i rows: every kept off-diagonal block costs 4 * n_i * B * d
    (QK^T and PV), the diagonal block 2 * n_i^2 * d (its causal half). Dense-equivalent: 2 * d * L^2
    per head and sequence. At tau <= 0 the two agree.
    """
    eff = 0.0
    dense = 0.0
    gb = 0
    hq = counts.shape[0]
    for s in range(len(cu) - 1):
        L = int(cu[s + 1] - cu[s])
        nb = (L + B - 1) // B
        if nb == 0:
            continue
        n = np.minimum(B, L - np.arange(nb) * B).astype(np.float64)
        c = counts[:, gb:gb + nb].astype(np.float64)
        eff += float((4.0 * d * (c - 1) * n[None, :] * B).sum() + hq * (2.0 * d * n * n).sum())
        dense += 2.0 * d * hq * float(L) * float(L)
        gb += nb
    return eff, dense


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return self.summary()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if len(r) > 8 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) > 8 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            if len(r) > 8:
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.rows)}


def workload(args):
    w = synth.WORKLOADS[args.workload]
    if args.lens:
        lens = [int(v) for v in args.lens.split(",")]
        w = w.with_lens(lens, seeds=list(w.seeds[: len(lens)]) + list(range(len(w.seeds), len(lens))),
                        name=f"{w.name}@lens={args.lens}")
    return w


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def replica_workload(w, rank: int):
    """The workload of one replica: same shapes, rank-distinct seeds (rank 0 keeps the originals)."""
    return w if rank == 0 else w.with_lens(w.lens, seeds=[s + 1000 * rank for s in w.seeds])


def reduce_over_ranks(work: list[float], times: list[float], dist=None, device="cpu"):
    """Whole-job totals of a replica run: the work units summed over ranks and the timings maxed over
    ranks (every rank calls this once, with lists of the same lengths, so the collectives match)."""
    if dist is None:
        return list(work), list(times)
    import torch
    w = torch.tensor(work, dtype=torch.float64, device=device)
    t = torch.tensor(times, dtype=torch.float64, device=device)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return w.tolist(), t.tolist()


def supplementary(fp, p, sp, x, q, k, v, tau, stream, w, reps=3):
    """Outside the timed step: (1) the cumulative top-p selector (the selection FlashPrefill's max
    threshold replaces) against the threshold search alone, on the same pooled tensors; (2) FP8
    attention (e4m3 Q / K with per-tensor scales, bf16 V) on the step's own lists."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    out = {}
    counts2 = torch.zeros_like(sp.counts)
    idx2 = torch.zeros_like(sp.indices)
    scores = torch.empty(max(p.index_elems, 1), dtype=torch.float32, device="cuda")
    gamma = 0.95
    out["threshold_search_ms"] = round(timed(lambda: fp.block_search(p, sp.q_pool, sp.k_pool, tau, counts2, idx2,
                                                                        sp.dev_status, stream)), 4)
    out["topp_search_ms"] = round(timed(lambda: fp.block_search_topp(p, sp.q_pool, sp.k_pool, gamma, scores, counts2,
                                                                        idx2, sp.dev_status, stream)), 4)
    eff, dense = kept_flops(counts2[:, : p.total_blocks].cpu().numpy(), x["cu_seqlens"], w.block, w.d)
    out["topp_gamma"] = gamma
    out["topp_density"] = round(eff / dense, 6)
    out["topp_scores_bytes"] = int(4 * p.index_elems)
    del scores, counts2, idx2
    # FP8: per-tensor scales from the absolute maxima, e4m3 codes quantised on the host
    q32, k32 = synth.bf16_bits_to_f32(x["q"]), synth.bf16_bits_to_f32(x["k"])
    qs, ks = float(np.abs(q32).max()) / 448.0, float(np.abs(k32).max()) / 448.0
    qc = torch.from_numpy(synth.to_e4m3_bits(q32 / qs)).cuda()
    kc = torch.from_numpy(synth.to_e4m3_bits(k32 / ks)).cuda()
    del q32, k32
    o8 = torch.empty_like(sp.out)
    ms8 = timed(lambda: fp.block_sparse_attn_fp8(p, qc, kc, v, qs, ks, sp.counts, sp.indices, 0.0, o8, None,
                                                 sp.dev_status, stream))
    eff1, _ = kept_flops(sp.counts[:, : p.total_blocks].cpu().numpy(), x["cu_seqlens"], w.block, w.d)
    out["fp8_attn_ms"] = round(ms8, 3)
    out["fp8_attn_tflops"] = round(eff1 / (ms8 * 1e-3) / 1e12, 2)
    out["fp8_note"] = "e4m3 Q K^T (kind::f8f6f4), bf16 P V; effective FLOPs of the kept blocks"
    # the per-block power-of-two scale entry point on the same codes, every block's exponent set to
    # the power of two nearest the per-tensor scale (so the logits, and with them the softmax's path
    # through the kernel, have the per-tensor run's magnitudes)
    qe = torch.full((p.total_blocks, w.hq), int(round(math.log2(qs))), dtype=torch.int8, device="cuda")
    ke = torch.full((p.total_blocks, w.hkv), int(round(math.log2(ks))), dtype=torch.int8, device="cuda")
    msb = timed(lambda: fp.block_sparse_attn_fp8_blockscaled(p, qc, kc, v, qe, ke, sp.counts, sp.indices, 0.0, o8,
                                                             None, sp.dev_status, stream))
    out["fp8_blockscaled_attn_ms"] = round(msb, 3)
    out["fp8_blockscaled_attn_tflops"] = round(eff1 / (msb * 1e-3) / 1e12, 2)
    return out


def run_ours(args):
    import torch

    import block_sparse_long_causal_b200 as fp
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))

    w = workload(args)
    tau = w.tau if args.tau is None else args.tau
    w = replica_workload(w, rank)  # independent replica per rank: distinct seeds
    x = synth.make_inputs(w)
    cu = x["cu_seqlens"]
    p = fp.problem(cu, w.hq, w.hkv, w.d, w.block)
    sp = fp.SparsePrefill(p)

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)

    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(evs=None, tau=tau):
        # pool, search and sparse attention: three C-ABI calls, one kernel each, an event between them
        if evs:
            evs[0].record(stream)
        fp.block_pool(p, q, k, sp.q_pool, sp.k_pool, stream)
        if evs:
            evs[1].record(stream)
        fp.block_search(p, sp.q_pool, sp.k_pool, tau, sp.counts, sp.indices, sp.dev_status, stream)
        if evs:
            evs[2].record(stream)
        fp.block_sparse_attn(p, q, k, v, sp.counts, sp.indices, 0.0, sp.out, None, sp.dev_status, stream)
        if evs:
            evs[3].record(stream)

    def dense():
        fp.dense_attn(p, q, k, v, 0.0, sp.out, None, sp.dev_status, stream)

    def interleaved(n, tau):
        """n (sparse step, dense attention) pairs launched back to back, so that the two kernels of a
        pair see the same clock and power state. Returns per-pair step and dense times (ms)."""
        il = [[ev() for _ in range(5)] for _ in range(n)]
        for e in il:
            step(e, tau)  # records e[0] .. e[3]
            dense()
            e[4].record(stream)
        torch.cuda.synchronize()
        return ([e[0].elapsed_time(e[3]) for e in il], [e[3].elapsed_time(e[4]) for e in il],
                [e[0].elapsed_time(e[1]) for e in il], [e[1].elapsed_time(e[2]) for e in il],
                [e[2].elapsed_time(e[3]) for e in il])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(sp.dev_status.item()) == 0, "device status after warm-up"

    # dense baseline (own kernel, same design) for the speedup: interleaved with the sparse step
    # (pool + search, then the sparse attention) launch by launch, so that both see the same clock
    # and power state (a short kernel timed first runs at a higher clock under the power cap)
    dense_ms = step_il_ms = ratio = None
    if not args.no_dense:
        for _ in range(2):
            dense()
        torch.cuda.synchronize()
        st_il, de_il, _, _, _ = interleaved(max(3, args.steps), tau)
        step_il_ms, dense_ms = float(np.median(st_il)), float(np.median(de_il))
        r = [d / s_ for d, s_ in zip(de_il, st_il)]
        ratio = {"median": round(float(np.median(r)), 4), "min": round(min(r), 4), "max": round(max(r), 4),
                 "pairs": len(r)}

    supp = None if args.no_supplementary else supplementary(fp, p, sp, x, q, k, v, tau, stream, w)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    events = [[ev() for _ in range(4)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for i in range(args.steps):
        step(events[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    pool_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in events]))
    search_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in events]))
    attn_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in events]))
    status = int(sp.dev_status.item())

    counts = sp.counts[:, : p.total_blocks].cpu().numpy()
    eff_flops, dense_flops = kept_flops(counts, cu, w.block, w.d)
    density = eff_flops / dense_flops
    pk = peaks()

    # ---- labelled supplementary thresholds (outside the timed step): the same workload at tau values
    # where the search drops blocks, each step interleaved with the dense kernel for the speedup
    sparse_settings = []
    if not args.no_dense and args.sparse_taus:
        for tau_s in [float(t) for t in args.sparse_taus.split(",")]:
            for _ in range(2):
                step(None, tau_s)
            torch.cuda.synchronize()
            st_il, de_il, po_il, se_il, at_il = interleaved(max(3, args.sparse_pairs), tau_s)
            # the same sparse steps back to back (no dense launch between them): the kernel at the
            # clock its own load settles to under the power cap
            bb = [[ev() for _ in range(4)] for _ in range(max(3, args.sparse_pairs))]
            for e in bb:
                step(e, tau_s)
            torch.cuda.synchronize()
            at_bb = float(np.median([e[2].elapsed_time(e[3]) for e in bb]))
            c_s = sp.counts[:, : p.total_blocks].cpu().numpy()
            eff_s, _ = kept_flops(c_s, cu, w.block, w.d)
            at_ms = float(np.median(at_il))
            r = [d / s_ for d, s_ in zip(de_il, st_il)]
            tf = eff_s / (at_ms * 1e-3) / 1e12
            sparse_settings.append({
                "tau": tau_s, "label": "supplementary (workload threshold is %g)" % tau,
                "density": round(eff_s / dense_flops, 6), "effective_tflop": round(eff_s / 1e12, 4),
                "step_ms": round(float(np.median(st_il)), 4), "pool_ms": round(float(np.median(po_il)), 4),
                "search_ms": round(float(np.median(se_il)), 4), "attn_ms": round(at_ms, 4),
                "dense_ms": round(float(np.median(de_il)), 4), "attn_tflops": round(tf, 2),
                "attn_frac_sustained": round(tf / pk["bf16_tflops_sustained"], 4),
                "attn_frac_burst": round(tf / pk["bf16_tflops"], 4),
                "attn_ms_back_to_back": round(at_bb, 4),
                "attn_frac_sustained_back_to_back": round(eff_s / (at_bb * 1e-3) / 1e12 / pk["bf16_tflops_sustained"], 4),
                "speedup_vs_own_dense": {"median": round(float(np.median(r)), 4), "min": round(min(r), 4),
                                         "max": round(max(r), 4), "pairs": len(r)}})
        step(None, tau)  # leave the workload's own lists in place
        torch.cuda.synchronize()

    # ---- e2e through the C ABI with host buffers (H2D of Q/K/V and D2H of O inside the timed region)
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (torch.from_numpy(a.view(np.int16)).pin_memory() for a in (x["q"], x["k"], x["v"]))
        oh = torch.empty((p.total_tokens, w.hq, w.d), dtype=torch.int16).pin_memory()
        # a prefill stream as a server runs it: step i's inputs go host -> device on one copy stream
        # and step i - 1's output device -> host on another while step i - 1 computes, so two device
        # slots of inputs and outputs alternate; every step's copies and its one-call prefill
        # (fp_sparse_prefill, the public API) lie inside the timed region
        slots_in = [(q, k, v), (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))]
        slots_out = [sp.out, torch.empty_like(sp.out)]
        s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
        workspace = torch.empty(fp.sparse_prefill_workspace(p), dtype=torch.uint8, device="cuda")
        n_e2e = max(2, args.steps)

        def e2e_run(n, first_ev=None, last_ev=None):
            ev_in, ev_comp, ev_out = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
            if first_ev is not None:
                first_ev.record(s_h2d)
            for i in range(n):
                sl = i % 2
                qd, kd, vd = slots_in[sl]
                with torch.cuda.stream(s_h2d):
                    if i >= 2:
                        s_h2d.wait_event(ev_comp[i - 2])  # the slot's previous step has read its inputs
                    for dst, src in ((qd, qh), (kd, kh), (vd, vh)):
                        dst.view(torch.int16).copy_(src, non_blocking=True)
                    ev_in[i].record(s_h2d)
                stream.wait_event(ev_in[i])
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])  # the slot's previous output is back on the host
                fp.sparse_prefill(p, qd, kd, vd, tau, 0.0, workspace, slots_out[sl], None, sp.dev_status, stream)
                ev_comp[i].record(stream)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(ev_comp[i])
                    oh.copy_(slots_out[sl][: p.total_tokens].view(torch.int16), non_blocking=True)
                    ev_out[i].record(s_d2h)
            if last_ev is not None:
                last_ev.record(s_d2h)

        e2e_run(2)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a0, a1 = ev(), ev()
        e2e_run(n_e2e, a0, a1)
        torch.cuda.synchronize()
        e2e_ms = a0.elapsed_time(a1) / n_e2e
        h2d = sum(a.nbytes for a in (x["q"], x["k"], x["v"]))
        d2h = oh.numel() * 2
        e2e = {"ms": e2e_ms, "h2d": h2d, "d2h": d2h}

    # whole job: kept-block FLOPs summed over ranks, times maxed over ranks
    ms_step = total_ms / args.steps
    (job_flops,), (ms_step, attn_ms, pool_ms, search_ms, e2e_max, dense_ms_max, step_il_max) = reduce_over_ranks(
        [eff_flops], [ms_step, attn_ms, pool_ms, search_ms, e2e["ms"] if e2e else 0.0, dense_ms or 0.0,
                      step_il_ms or 0.0],
        dist, device="cuda")
    if e2e:
        e2e["ms"] = e2e_max
    if dense_ms is not None:
        dense_ms, step_il_ms = dense_ms_max, step_il_max

    peak_tf = pk["bf16_tflops_sustained"]
    attn_tflops = eff_flops / (attn_ms * 1e-3) / 1e12
    value = job_flops / (ms_step * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "seq_lens": list(w.lens), "num_q_heads": w.hq, "num_kv_heads": w.hkv,
            "head_dim": w.d, "block": w.block, "tau": tau, "global_batch": len(w.lens) * ws,
            "seq_len": int(max(w.lens)), "parallelism": f"replicas{ws}",
            "l2": "inputs (Q+K+V %.2f GB) larger than L2; no flush" % (sum(a.nbytes for a in (x['q'], x['k'], x['v'])) / 1e9),
        },
        "breakdown_ms": {"pool": round(pool_ms, 4), "search": round(search_ms, 4), "sparse_attn": round(attn_ms, 4),
                         "dense_attn": round(dense_ms, 4) if dense_ms else None},
        "sparse_prefill_ms": round(ms_step, 4),
        "effective_tflop": round(eff_flops / 1e12, 4),
        "dense_equiv_tflop": round(dense_flops / 1e12, 4),
        "density": round(density, 6),
        # dense attention over the sparse step (pool + search + sparse attention), timed interleaved:
        # the median of the per-pair ratios, with their range
        "speedup_vs_own_dense": ratio["median"] if ratio else None,
        "speedup_vs_own_dense_range": ratio,
        "roofline": {"bound": "tensor", "kernel": "sparse_attn", "achieved": round(attn_tflops, 2),
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(attn_tflops / peak_tf, 4),
                     "peak_source": f"{pk['source']} bf16 sustained",
                     "peak_burst": pk["bf16_tflops"], "frac_of_burst": round(attn_tflops / pk["bf16_tflops"], 4),
                     "traffic": measured_traffic(f"attn_kernel<{w.block}>", w.name)},
        "search_roofline": None,
        "sparse_settings": sparse_settings,
        # per step: pool_kernel, (ksplit_kernel with the problem's key split,) search_kernel, attn_kernel
        # and, for B = 128, attn_rows_kernel (one of the two attention kernels returns at once)
        "gpu_launches": (3 + (p.key_split is not None) + (w.block == 128)) * args.steps,
        "supplementary": supp,
        "dev_status": status,
        "clocks": clk,
    }
    # search (pool + threshold + lists) against HBM: algorithmic bytes = read Q, K; write and read
    # the pooled tensors; write counts and the kept indices
    T, NB = p.total_tokens, p.total_blocks
    search_bytes = (2 * T * (w.hq + w.hkv) * w.d + 2 * 4 * NB * (w.hq + w.hkv) * w.d
                    + 4 * w.hq * NB + 4 * float(counts.sum()))
    s_ms = pool_ms + search_ms
    # per kernel: pool reads Q and K and writes the pooled tensors; search reads the pooled tensors
    # and writes the counts and the kept indices
    pool_bytes = 2 * T * (w.hq + w.hkv) * w.d + 4 * NB * (w.hq + w.hkv) * w.d
    srch_bytes = 4 * NB * (w.hq + w.hkv) * w.d + 4 * w.hq * NB + 4 * float(counts.sum())
    gbs = lambda b, ms: round(b / (ms * 1e-3) / 1e9, 1)  # noqa: E731
    line["search_roofline"] = {"bound": "hbm", "kernels": "pool_kernel + search_kernel",
                               "achieved": gbs(search_bytes, s_ms),
                               "peak": pk["hbm_gbs"], "unit": "GB/s",
                               "frac": round(search_bytes / (s_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                               "bytes": search_bytes,
                               "pool_kernel": {"ms": round(pool_ms, 4), "bytes": pool_bytes,
                                               "achieved": gbs(pool_bytes, pool_ms),
                                               "frac": round(gbs(pool_bytes, pool_ms) / pk["hbm_gbs"], 4)},
                               "search_kernel": {"ms": round(search_ms, 4), "bytes": srch_bytes,
                                                 "achieved": gbs(srch_bytes, search_ms),
                                                 "frac": round(gbs(srch_bytes, search_ms) / pk["hbm_gbs"], 4)}}
    if e2e:
        line["e2e"] = {"value": round(job_flops / (e2e["ms"] * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                       "ms_per_step": round(e2e["ms"], 3), "h2d_bytes_per_step": e2e["h2d"],
                       "d2h_bytes_per_step": e2e["d2h"],
                       "copies": "step i+1 host->device and step i-1 device->host on two copy streams during "
                                 "step i's fp_sparse_prefill (two device slots); %d steps" % n_e2e}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, tau, budget_s=args.cpu_budget)
    if dist:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_baseline(w, tau, budget_s=20.0, x=None):
    """The fp64 oracle on a bounded sample of the workload, scaled to effective TFLOP/s.

    Full pool + search on the whole workload, then exact attention on a seeded sample of
    (token, head) rows (grown until about budget_s seconds of attention work). The full-workload
    time is estimated as search time + sample time * (total attended pairs / sampled pairs).
    """
    import oracle
    if x is None:
        x = synth.make_inputs(w)
    cu = x["cu_seqlens"]
    t0 = time.perf_counter()
    qb, kb = oracle.pool(x["q"], cu, w.block), oracle.pool(x["k"], cu, w.block)
    counts, idx, _ = oracle.search(qb, kb, cu, w.block, tau, want_band=False)
    t_search = time.perf_counter() - t0
    eff_flops, _ = kept_flops(counts, cu, w.block, w.d)
    rng = np.random.default_rng(0)
    T = int(cu[-1])
    pairs_total = 0.0  # exact attended (query, key) pairs of the whole prefill
    gb = 0
    for s in range(len(cu) - 1):
        L = int(cu[s + 1] - cu[s])
        nb = (L + w.block - 1) // w.block
        nrow = np.minimum(w.block, L - np.arange(nb) * w.block).astype(np.float64)
        c = counts[:, gb:gb + nb].astype(np.float64)
        pairs_total += float(((c - 1) * nrow[None, :] * w.block).sum() + w.hq * (nrow * (nrow + 1) / 2).sum())
        gb += nb
    n, t_attn, pairs = 16, 0.0, 0.0
    while True:
        tok = rng.integers(0, T, n).astype(np.int64)
        head = rng.integers(0, w.hq, n).astype(np.int32)
        t1 = time.perf_counter()
        oracle.attn_rows(x["q"], x["k"], x["v"], cu, w.block, tok, head, counts, idx)
        t_attn += time.perf_counter() - t1
        # attended pairs of the sampled rows (kept blocks up to the row's position)
        for t, h in zip(tok, head):
            s = int(np.searchsorted(cu, t, side="right") - 1)
            pos = int(t - cu[s])
            i = pos // w.block
            gb = oracle.block_base(cu, w.block, s) + i
            c = int(counts[h, gb])
            pairs += (c - 1) * w.block + (pos - i * w.block + 1)
        if t_attn >= budget_s * 0.5 or n >= 4096:
            break
        n *= 2
    est_s = t_search + t_attn * pairs_total / max(pairs, 1.0)
    return {"value": round(eff_flops / est_s / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": (f"fp64 oracle: full pool+search of {w.name} ({t_search:.1f} s), exact attention on "
                       f"{int(n * 2 - 16)} seeded (token, head) rows ({t_attn:.1f} s, {pairs:.3g} of "
                       f"{pairs_total:.3g} attended pairs), extrapolated to the whole prefill"),
            "est_full_prefill_s": round(est_s, 1), "nproc": os.cpu_count()}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    w = workload(args)
    tau = w.tau if args.tau is None else args.tau
    x = synth.make_inputs(w)
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, tau, budget_s=budget, x=x)
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(w, tau, budget_s=budget, x=x)
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    value = float(np.mean(vals))
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * wall / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "seq_lens": list(w.lens), "num_q_heads": w.hq, "num_kv_heads": w.hkv,
                       "head_dim": w.d, "block": w.block, "tau": tau, "global_batch": len(w.lens),
                       "seq_len": int(max(w.lens)), "parallelism": "cpu"},
            "cpu_baseline": dict(last, value=round(value, 6)),
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(synth.WORKLOADS))
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--lens", type=str, default=None,
                    help="comma-separated sequence lengths replacing the workload's (smaller case of the same shape)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-supplementary", action="store_true",
                    help="skip the top-p comparison and FP8 timings reported beside the step")
    ap.add_argument("--sparse-taus", type=str, default="0.95,0.98",
                    help="comma-separated supplementary thresholds reported beside the workload's own ('' for none)")
    ap.add_argument("--sparse-pairs", type=int, default=7,
                    help="interleaved (sparse step, dense) pairs per supplementary threshold")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
