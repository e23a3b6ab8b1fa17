"""Benchmark of the M-FALCON prefill + pool write + rank decode path on B200.

One step = one single-layer pass of the whole path over one synthetic batch:
  1. pool write: the past K/V of every user into its slot of the pool,
  2. masked prefill attention over [n past || k candidates] for every user,
  3. rank decode of the same candidates over the pool (past rows + self).
Default workload: 256 users, n ~ U{32..4096}, k ~ U{50..2000}, H=8, D=128,
pool [L=1, S=256, H=8, n_cap=4096, D=128] (the ragged mixed batch).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
Prints ONE JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kv_cache_reuse_falcon_b200 import synth  # noqa: E402
from kv_cache_reuse_falcon_b200.shard import combine_rank_results, rank_seed, segment_cost  # noqa: E402

DEFAULT_WORKLOAD = "ragged_B256_H8_D128_n32-4096_k50-2000"
METRIC = "candidate tokens scored/s + prefill TFLOP/s (mask-effective) & decode HBM GB/s"


# ---------------------------------------------------------------- accounting

def prefill_flops(past, cand, H, D):
    """Mask-effective FLOPs: 4*D per allowed score entry (QK^T and PV), all heads."""
    return float(4.0 * D * H * segment_cost(past, cand).sum())


def decode_flops(past, cand, H, D):
    """Each candidate row scores n_r pool keys plus itself."""
    p = np.asarray(past, dtype=np.float64)
    k = np.asarray(cand, dtype=np.float64)
    return float(4.0 * D * H * (k * (p + 1)).sum())


def decode_bytes(past, cand, H, D, out_bytes, pool_elem_bytes=2):
    """Algorithmic bytes: pool K/V rows read once + candidate q/k/v read + output written."""
    p = np.asarray(past, dtype=np.float64).sum()
    k = np.asarray(cand, dtype=np.float64).sum()
    return float(2 * p * H * D * pool_elem_bytes + 3 * k * H * D * 2 + k * H * D * out_bytes)


def prefill_bytes(T, H, D, out_bytes):
    return float(3 * T * H * D * 2 + T * H * D * out_bytes)


def pool_write_bytes(past, H, D):
    return float(2 * 2 * np.asarray(past, dtype=np.float64).sum() * H * D * 2)   # K and V, read + write


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the prefill
# attention kernel per query-side token, from one ncu capture of a 24-user cut
# of the ragged batch (H=8, D=128; summary and command under profiles/), keyed
# by the kernel source it was taken on.  A changed kernel reports null until
# it is captured again.
_PREFILL_TRAFFIC_PER_TOKEN = {
    # kernel_source_key() of csrc/attn_sm100.cuh, H, D: bytes per token (reads + writes,
    # the writes including the fused store of the past K/V into the pool)
    ("1b9929abd9486744", 8, 128): (432.074752e6 + 292.394496e6) / 70236,
}


def kernel_source_key(path=None):
    """sha256 prefix of the attention kernel's code with comments and blank
    space removed: what the captured counters depend on."""
    import hashlib
    import re
    path = path or os.path.join(ROOT, "kv_cache_reuse_falcon_b200", "csrc", "attn_sm100.cuh")
    with open(path) as f:
        text = f.read()
    code = re.sub(r"/\*.*?\*/", "", re.sub(r"//[^\n]*", "", text), flags=re.S)
    code = "\n".join(" ".join(ln.split()) for ln in code.splitlines() if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def prefill_traffic(T, H, D):
    per = _PREFILL_TRAFFIC_PER_TOKEN.get((kernel_source_key(), H, D))
    return None if per is None else per * T


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------- workload

def make_workload(name: str, seed: int, users: int = 0):
    """Host arrays of one step's inputs (bf16 bits) for the named workload.

    users > 0 replaces the workload's user count (and pool slot count) to make a
    smaller case of the same length distribution, e.g. for profiler captures."""
    w = synth.workload(name)
    if users > 0:
        import dataclasses
        w = dataclasses.replace(w, B=users, S=users)
    rng = np.random.Generator(np.random.PCG64(seed))
    past, cand = w.lengths(rng)
    S = w.S if w.S else max(w.B, 1)
    batch = synth.make_prefill(seed, past, cand, w.H, w.D, n_slots=S, rng=rng)
    n_cap = w.n_cap if w.n_cap else int(past.max())
    return w, batch, S, n_cap


def candidate_index(batch):
    return np.concatenate([np.arange(batch.cu_seqlens[b] + batch.past_lens[b], batch.cu_seqlens[b + 1])
                           for b in range(batch.B)]).astype(np.int64)


# ------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples over the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def _lines(self):
        try:
            with open(self.path) as f:
                return [ln for ln in f.read().splitlines() if ln.count(",") >= 8]
        except OSError:
            return []

    def start(self):
        """Start sampling every 50 ms; returns once the first sample is in (at most 5 s), so the
        timed region that follows is covered from its start."""
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w", buffering=1)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 5.0 and not self._lines():
            time.sleep(0.01)
        self.first = len(self._lines())   # samples before the timed region are not used

    def stop(self):
        """Waits for one sample after the timed region (at most 1 s), then stops sampling and
        summarises the samples taken from the start of the timed region on."""
        if self.proc is None:
            return None
        n_end = len(self._lines())
        t0 = time.time()
        while time.time() - t0 < 1.0 and len(self._lines()) <= n_end:
            time.sleep(0.01)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self._lines()[self.first:]:
            parts = [x.strip() for x in line.split(",")]
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ oracle timing

def cpu_oracle_sample(batch, n_cap_unused=None, budget_s: float = 12.0, max_segments: int = 64, seed: int = 0):
    """Time the CPU oracle on a bounded sample of users (prefill of all rows + decode of the candidates)."""
    import oracle
    rng = np.random.default_rng(seed)
    order = rng.permutation(batch.B)
    done_cand = 0
    t_total = 0.0
    used = 0
    H, D = batch.H, batch.D
    for b in order[:max_segments]:
        lo, hi = int(batch.cu_seqlens[b]), int(batch.cu_seqlens[b + 1])
        n = int(batch.past_lens[b])
        q, k, v = batch.q[lo:hi], batch.k[lo:hi], batch.v[lo:hi]
        t0 = time.perf_counter()
        oracle.prefill(q, k, v, np.array([0, hi - lo], np.int32), np.array([n], np.int32))
        # decode of the same candidates over the segment's past rows (a one-slot pool)
        pk = np.ascontiguousarray(k[:n].transpose(1, 0, 2))[None, None]
        pv = np.ascontiguousarray(v[:n].transpose(1, 0, 2))[None, None]
        if n == 0:
            pk = np.zeros((1, 1, H, 1, D), np.uint16)
            pv = pk.copy()
        oracle.decode(q[n:], k[n:], v[n:], np.array([0, hi - lo - n], np.int32), np.array([0], np.int32),
                      np.array([n], np.int32), pk, pv, 0)
        t_total += time.perf_counter() - t0
        done_cand += hi - lo - n
        used += 1
        if t_total >= budget_s:
            break
    return {"value": done_cand / t_total, "unit": "candidate tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d of %d users (all their rows: prefill + pool-row decode of their candidates), "
                      "%.1f s of fp64 CPU work" % (used, batch.B, t_total),
            "seconds": t_total}


# ------------------------------------------------------------------ runner

def run_ours(args, rank, world, device, dist):
    import torch
    from kv_cache_reuse_falcon_b200 import binding as ub

    w = synth.workload(args.workload)
    name = w.name
    seed = rank_seed(w.seed, rank)
    w, batch, S, n_cap = make_workload(name, seed, args.users)
    H, D = batch.H, batch.D
    T = batch.T
    past, cand = batch.past_lens, batch.cand_lens
    cidx = candidate_index(batch)
    Tc = int(cidx.shape[0])

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    def dev_i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    q, k, v = dev_bf16(batch.q), dev_bf16(batch.k), dev_bf16(batch.v)
    qc, kc, vc = dev_bf16(batch.q[cidx]), dev_bf16(batch.k[cidx]), dev_bf16(batch.v[cidx])
    cu, pl, sl = dev_i32(batch.cu_seqlens), dev_i32(past), dev_i32(batch.slot_ids)
    cu_c = dev_i32(synth.cu_from_lens(cand))
    L = max(w.L, 1)
    pool_k = torch.full((L, S, H, n_cap, D), 0x7FC0, dtype=torch.int16, device=device).view(torch.bfloat16)
    pool_v = torch.full((L, S, H, n_cap, D), 0x7FC0, dtype=torch.int16, device=device).view(torch.bfloat16)
    out_p = torch.empty((T, H, D), dtype=torch.bfloat16, device=device)
    out_d = torch.empty((Tc, H, D), dtype=torch.bfloat16, device=device)
    max_seqlen = int(np.diff(batch.cu_seqlens).max())
    max_past = int(past.max())
    max_k = int(cand.max())
    ws_bytes = ub.rank_decode_workspace_size(batch.B, H, D, max_k, Tc, n_cap)
    ws = torch.empty(ws_bytes // 4 + 4, dtype=torch.float32, device=device)
    ws_pre = torch.empty(ub.masked_prefill_workspace_size() // 4 + 4, dtype=torch.float32, device=device)
    decode_split = ws_bytes > 256
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    layer = 0

    def step(ev=None):
        # the prefill also writes every user's past K/V into its pool slot (one kernel)
        if ev is not None:
            ev[0].record(stream)
        ub.masked_prefill_attn(q, k, v, cu, pl, max_seqlen, out=out_p, out_fp32=False, workspace=ws_pre,
                               pool_k=pool_k, pool_v=pool_v, slot_ids=sl, layer=layer, dev_status=status,
                               stream=stream)
        if ev is not None:
            ev[2].record(stream)
        ub.rank_decode_attn(qc, kc, vc, cu_c, sl, pl, pool_k, pool_v, layer, max_k, out=out_d, out_fp32=False,
                            workspace=ws, dev_status=status, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError("device status %s after warm-up" % ub.status_string(int(status.item())))

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    elapsed_ms = start.elapsed_time(stop)
    t_pre = [e[0].elapsed_time(e[2]) for e in evs]
    t_dec = [e[2].elapsed_time(e[3]) for e in evs]
    if int(status.item()) != 0:
        raise RuntimeError("device status %s in the timed region" % ub.status_string(int(status.item())))

    # ------------------------------------------------------ end to end (host buffers)
    # Every step copies its inputs (Q, K, V, the length / slot arrays and the
    # candidate row index) from pinned host memory on a copy stream into one of
    # two device buffer sets, so step i+1's copies run while step i computes;
    # the candidates' q/k/v are gathered on the device from the copied tensors,
    # and the decode output is read back into pinned host memory.
    hcidx = torch.from_numpy(cidx).pin_memory()
    hin = [torch.from_numpy(batch.q.view(np.int16)).pin_memory(),
           torch.from_numpy(batch.k.view(np.int16)).pin_memory(),
           torch.from_numpy(batch.v.view(np.int16)).pin_memory(),
           torch.from_numpy(batch.cu_seqlens.astype(np.int32)).pin_memory(),
           torch.from_numpy(past.astype(np.int32)).pin_memory(),
           torch.from_numpy(batch.slot_ids.astype(np.int32)).pin_memory(),
           torch.from_numpy(synth.cu_from_lens(cand)).pin_memory(),
           hcidx]
    hout = torch.empty((Tc, H, D), dtype=torch.bfloat16).pin_memory()
    sets = [[q.view(torch.int16), k.view(torch.int16), v.view(torch.int16), cu, pl, sl, cu_c,
             torch.empty_like(hcidx, device=device)],
            [torch.empty_like(h, device=device) for h in hin]]
    h2d_bytes = sum(h.numel() * h.element_size() for h in hin)
    d2h_bytes = hout.numel() * hout.element_size()
    e2e_steps = max(2, min(args.steps, 4))
    copy_stream = torch.cuda.Stream(device)
    ev_copied = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_used = [torch.cuda.Event() for _ in range(e2e_steps)]

    def e2e_step(i):
        dq, dk, dv, dcu, dpl, dsl, dcuc, dcidx = sets[i % 2]
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(ev_used[i - 2])     # step i-2 is done with this set
            for h, d in zip(hin, sets[i % 2]):
                d.copy_(h, non_blocking=True)
            ev_copied[i].record(copy_stream)
        stream.wait_event(ev_copied[i])
        torch.index_select(dq, 0, dcidx, out=qc.view(torch.int16))
        torch.index_select(dk, 0, dcidx, out=kc.view(torch.int16))
        torch.index_select(dv, 0, dcidx, out=vc.view(torch.int16))
        bq, bk, bv = dq.view(torch.bfloat16), dk.view(torch.bfloat16), dv.view(torch.bfloat16)
        ub.masked_prefill_attn(bq, bk, bv, dcu, dpl, max_seqlen, out=out_p, out_fp32=False, workspace=ws_pre,
                               pool_k=pool_k, pool_v=pool_v, slot_ids=dsl, layer=layer, dev_status=status,
                               stream=stream)
        ub.rank_decode_attn(qc, kc, vc, dcuc, dsl, dpl, pool_k, pool_v, layer, max_k, out=out_d, out_fp32=False,
                            workspace=ws, dev_status=status, stream=stream)
        hout.copy_(out_d, non_blocking=True)
        ev_used[i].record(stream)

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if int(status.item()) != 0:
        raise RuntimeError("device status %s in the end-to-end steps" % ub.status_string(int(status.item())))
    del sets

    # ---------------------------------------------------------- max over ranks
    times, counts = combine_rank_results(
        {"step": elapsed_ms / args.steps, "e2e": e2e_ms, "prefill": sum(t_pre) / len(t_pre),
         "decode": sum(t_dec) / len(t_dec)},
        {"candidates": float(cand.sum())}, group=dist.group.WORLD if dist is not None else False, device=device)
    ms_step, e2e_ms, pre_ms, dec_ms = (times[k] for k in ("step", "e2e", "prefill", "decode"))
    cand_total = counts["candidates"]

    peaks = load_peaks()
    pf = prefill_flops(past, cand, H, D)
    df = decode_flops(past, cand, H, D)
    db = decode_bytes(past, cand, H, D, 2)
    pre_tflops = pf / (pre_ms * 1e-3) / 1e12
    dec_tflops = df / (dec_ms * 1e-3) / 1e12
    dec_gbs = db / (dec_ms * 1e-3) / 1e9
    dec_roof = roof_entry(dec_ms, df, db, peaks, "decode")   # the decode's own binding roof
    # The prefill kernel runs for milliseconds inside a sub-second timed region at
    # full clock, so the burst GEMM figure is its denominator (the stricter one).
    peak = peaks["bf16_tflops"]
    result = {
        "metric": METRIC,
        "value": cand_total / (ms_step * 1e-3),
        "unit": "candidate tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": name if not args.users else "%s[users=%d]" % (name, args.users),
                   "users_per_gpu": batch.B, "H": H, "D": D,
                   "tokens_per_gpu": T, "candidates_per_gpu": Tc, "pool": [L, S, H, n_cap, D],
                   "layers_per_step": 1, "parallelism": "users sharded across %d GPU(s), no collective" % world,
                   "l2": "inputs larger than L2 (no flush)", "seed_rank0": seed},
        "phases": {"prefill_ms": pre_ms, "decode_ms": dec_ms, "prefill_writes_pool": True,
                   "prefill_tflops": pre_tflops, "decode_tflops": dec_tflops, "decode_gbs": dec_gbs,
                   "prefill_frac_tensor": pre_tflops / peak,
                   "prefill_frac_tensor_sustained": pre_tflops / peaks["bf16_tflops_sustained"],
                   "decode_frac_hbm": dec_gbs / peaks["hbm_gbs"],
                   "decode_bound": dec_roof["bound"], "decode_frac_roof": dec_roof["frac_roof"]},
        "roofline": {"kernel": "attn_fwd_kernel<128,prefill>", "bound": "tensor", "achieved": pre_tflops,
                     "peak": peak, "unit": "TFLOP/s", "frac": pre_tflops / peak,
                     "traffic": prefill_traffic(T, H, D),
                     "traffic_note": "ncu DRAM bytes per token of a 24-user capture, scaled by tokens",
                     "peak_source": "%s bf16_tflops (burst)" % peaks["source"],
                     "work_per_launch": "4*D*H*sum_b[n_b(n_b+1)/2 + k_b(n_b+1)] = %.4g FLOP" % pf},
        "e2e": {"value": cand_total / (e2e_ms * 1e-3), "unit": "candidate tokens/s",
                "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes),
                "steps": e2e_steps,
                "note": "inputs copied from pinned host memory on a second stream (double-buffered), "
                        "candidate rows gathered on the device, decode output read back"},
        "gpu_launches": args.steps * (2 + (1 if decode_split else 0)),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_oracle_sample(batch, budget_s=args.cpu_budget)
    if world == 1 and not args.no_sweep:
        del q, k, v, qc, kc, vc, pool_k, pool_v, out_p, out_d, ws, ws_pre
        torch.cuda.empty_cache()
        result["sweep"] = run_sweep(device, peaks)
    return result


def roof_entry(ms, flops, nbytes, peaks, kernel):
    """Rates of one timed call and its fraction of the roof that binds it (tensor or HBM)."""
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if t_tc >= t_hbm else "hbm"
    return {"kernel": kernel, "ms": ms, "tflops": tflops, "gbs": gbs, "bound": bound,
            "frac_tensor": tflops / peaks["bf16_tflops"], "frac_hbm": gbs / peaks["hbm_gbs"],
            "frac_roof": (t_tc if bound == "tensor" else t_hbm) * 1e3 / ms}


def run_sweep(device, peaks, iters=10, warm=3):
    """The other workloads, one GPU: the D=64 prefills and the rank decode from the L=12 pool
    at candidate counts 1..1000.  Inputs are N(0,1) bf16 drawn on the device from a seeded
    generator; L2 is flushed (a 256 MB write) before every timed call; each entry is the
    median over `iters` calls timed with CUDA events on the launching stream."""
    import torch
    from kv_cache_reuse_falcon_b200 import binding as ub

    stream = torch.cuda.current_stream(device)
    gen = torch.Generator(device=device)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=device)

    def randn(shape, seed):
        gen.manual_seed(seed)
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)

    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(iters):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(statistics.median(ts))

    status = torch.zeros(1, dtype=torch.int32, device=device)
    out = {}
    for key, wname in (("prefill_B64_n256_k128_D64", "prefill_B64"),
                       ("prefill_pool_B128_n1024_k512_D64", "prefill_pool_B128"),
                       ("table2_B8_n992_k656_D64", "table2_B8")):
        w = synth.workload(wname)
        past = np.full(w.B, w.n, np.int32)
        cand = np.full(w.B, w.k, np.int32)
        T = int((past + cand).sum())
        q, k, v = randn((T, w.H, w.D), w.seed), randn((T, w.H, w.D), w.seed + 1), randn((T, w.H, w.D), w.seed + 2)
        cu = torch.from_numpy(synth.cu_from_lens(past + cand)).to(device)
        pl = torch.from_numpy(past).to(device)
        o = torch.empty((T, w.H, w.D), dtype=torch.bfloat16, device=device)
        ws = torch.empty(ub.masked_prefill_workspace_size() // 4 + 4, dtype=torch.float32, device=device)
        kw = {}
        nbytes = prefill_bytes(T, w.H, w.D, 2)
        if w.L:
            pk = torch.zeros((w.L, w.S, w.H, w.n_cap, w.D), dtype=torch.bfloat16, device=device)
            pv = torch.zeros_like(pk)
            gen.manual_seed(w.seed + 3)
            slots = torch.randperm(w.S, generator=gen, device=device)[: w.B].to(torch.int32)
            kw = dict(pool_k=pk, pool_v=pv, slot_ids=slots, layer=0)
            nbytes += pool_write_bytes(past, w.H, w.D)

        def fn():
            ub.masked_prefill_attn(q, k, v, cu, pl, int(w.n + w.k), out=o, out_fp32=False, workspace=ws,
                                   dev_status=status, stream=stream, **kw)

        ms = timed(fn)
        e = roof_entry(ms, prefill_flops(past, cand, w.H, w.D), nbytes, peaks,
                       "attn_fwd_kernel<%d,prefill>%s" % (w.D, " (pool write fused)" if w.L else ""))
        e["candidates_per_s"] = float(cand.sum()) / (ms * 1e-3)
        out[key] = e
        del q, k, v, o, kw
        torch.cuda.empty_cache()

    # gradients of the prefill workload (B=64, n=256, k=128) at D=64 and D=128: forward with its
    # row statistic once, then the backward call timed; FLOPs = 10*D per allowed pair (S, dP,
    # dV, dK, dQ products)
    w = synth.workload("prefill_B64")
    past = np.full(w.B, w.n, np.int32)
    cand = np.full(w.B, w.k, np.int32)
    T = int((past + cand).sum())
    cu = torch.from_numpy(synth.cu_from_lens(past + cand)).to(device)
    pl = torch.from_numpy(past).to(device)
    for D in (64, 128):
        q, k, v, g = (randn((T, w.H, D), w.seed + j) for j in range(4))
        lse = torch.empty((T, w.H), dtype=torch.float32, device=device)
        o = ub.masked_prefill_attn(q, k, v, cu, pl, w.n + w.k, out_fp32=False, lse=lse, dev_status=status)
        grads = [torch.empty((T, w.H, D), dtype=torch.float32, device=device) for _ in range(3)]
        wsb = torch.empty(ub.masked_prefill_bwd_workspace_size(T, w.H) // 4 + 4, dtype=torch.float32,
                          device=device)

        def fn_bwd():
            ub.masked_prefill_bwd(q, k, v, o, g, lse, cu, pl, w.n + w.k, dq=grads[0], dk=grads[1], dv=grads[2],
                                  workspace=wsb, dev_status=status, stream=stream)

        ms = timed(fn_bwd)
        flops = 2.5 * prefill_flops(past, cand, w.H, D)
        nbytes = 5 * T * w.H * D * 2 + 3 * T * w.H * D * 4 + 2 * T * w.H * 4
        e = roof_entry(ms, flops, nbytes, peaks, "bwd_prep_kernel<%d> + bwd_kv_kernel<%d>" % (D, D))
        out["backward_B64_n256_k128_D%d" % D] = e
        del q, k, v, g, o, grads, lse

    # rank decode from the [12, 256, 8, 2048, 64] pool, 32 requests, every layer per step
    w = synth.workload("decode_R32")
    pk = randn((w.L, w.S, w.H, w.n_cap, w.D), w.seed)
    pv = randn((w.L, w.S, w.H, w.n_cap, w.D), w.seed + 1)
    gen.manual_seed(w.seed + 2)
    slots = torch.randperm(w.S, generator=gen, device=device)[: w.B].to(torch.int32)
    past = np.full(w.B, w.n, np.int32)
    pl = torch.from_numpy(past).to(device)
    for kk in (1, 16, 64, 128, 256, 1000):
        cand = np.full(w.B, kk, np.int32)
        Tc = int(cand.sum())
        cu = torch.from_numpy(synth.cu_from_lens(cand)).to(device)
        qkv = [[randn((Tc, w.H, w.D), w.seed + 10 * l + j) for j in range(3)] for l in range(w.L)]
        outs = [torch.empty((Tc, w.H, w.D), dtype=torch.bfloat16, device=device) for _ in range(w.L)]
        nws = ub.rank_decode_workspace_size(w.B, w.H, w.D, kk, Tc, w.n_cap)
        ws = torch.empty(nws // 4 + 4, dtype=torch.float32, device=device)

        def fn():
            for l in range(w.L):
                ub.rank_decode_attn(qkv[l][0], qkv[l][1], qkv[l][2], cu, slots, pl, pk, pv, l, kk, out=outs[l],
                                    out_fp32=False, workspace=ws, dev_status=status, stream=stream)

        ms = timed(fn) / w.L
        # the library sends requests of at most 64 candidates (one query head per kv head) to the small-k kernel
        kernel = ("decode_smallk_kernel<%d,%d>" % (w.D, 16 if kk <= 16 else 32 if kk <= 32 else 64)
                  if kk <= 64 else "attn_fwd_kernel<%d,decode>" % w.D)
        e = roof_entry(ms, decode_flops(past, cand, w.H, w.D), decode_bytes(past, cand, w.H, w.D, 2), peaks, kernel)
        e["candidates_per_s"] = float(Tc) / (ms * 1e-3)
        e["ms_per_12_layers"] = ms * w.L
        out["decode_R32_n2048_D64_k%d" % kk] = e
        del qkv, outs, ws
    del pk, pv
    torch.cuda.empty_cache()

    # the same decode from an E4M3 pool (codes of N(0, 1) / 0.0625 keys and values)
    scales = (0.0625, 0.0625)
    pk8 = (randn((w.L, w.S, w.H, w.n_cap, w.D), w.seed).float() / scales[0]).to(torch.float8_e4m3fn)
    pv8 = (randn((w.L, w.S, w.H, w.n_cap, w.D), w.seed + 1).float() / scales[1]).to(torch.float8_e4m3fn)
    for kk in (16, 64, 256):
        cand = np.full(w.B, kk, np.int32)
        Tc = int(cand.sum())
        cu = torch.from_numpy(synth.cu_from_lens(cand)).to(device)
        qkv = [[randn((Tc, w.H, w.D), w.seed + 10 * l + j) for j in range(3)] for l in range(w.L)]
        outs = [torch.empty((Tc, w.H, w.D), dtype=torch.bfloat16, device=device) for _ in range(w.L)]
        nws = ub.rank_decode_pool_workspace_size(pk8, pv8, w.B, w.H, kk, Tc, pool_scales=scales)
        ws = torch.empty(nws // 4 + 4, dtype=torch.float32, device=device)

        def fn8():
            for l in range(w.L):
                ub.rank_decode_attn(qkv[l][0], qkv[l][1], qkv[l][2], cu, slots, pl, pk8, pv8, l, kk, out=outs[l],
                                    out_fp32=False, workspace=ws, dev_status=status, stream=stream,
                                    pool_scales=scales)

        ms = timed(fn8) / w.L
        # the library's routing: the small-k kernel reads the codes in place up to 32 candidate
        # columns at D=64 (64 at D=128); beyond, a dequantized copy feeds the bfloat16 kernels
        if kk <= 32 or (w.D == 128 and kk <= 64):
            kernel = "decode_smallk_kernel<%d,%d,e4m3>" % (w.D, 16 if kk <= 16 else 32 if kk <= 32 else 64)
            path = "E4M3 codes expanded to bfloat16 in shared memory by the small-k kernel"
        elif kk <= 64:
            kernel = "kvpool_dequant_kernel + decode_smallk_kernel<%d,64>" % w.D
            path = "E4M3 rows dequantized into the workspace, then the bfloat16 small-k kernel"
        else:
            kernel = "kvpool_dequant_kernel + attn_fwd_kernel<%d,decode>" % w.D
            path = "E4M3 rows dequantized into the workspace, then the bfloat16 engine"
        e = roof_entry(ms, decode_flops(past, cand, w.H, w.D), decode_bytes(past, cand, w.H, w.D, 2, 1), peaks,
                       kernel)
        e["path"] = path
        e["candidates_per_s"] = float(Tc) / (ms * 1e-3)
        out["decode_R32_n2048_D64_k%d_e4m3" % kk] = e
        del qkv, outs, ws
    del pk8, pv8
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError("device status %s in the sweep" % ub.status_string(int(status.item())))
    del flush
    torch.cuda.empty_cache()
    return out


def run_decode_only(args, rank, world, device, dist):
    """Rank decode workload: R requests over an L-layer pool, one call per layer per step."""
    import torch
    from kv_cache_reuse_falcon_b200 import binding as ub

    w = synth.workload(args.workload)
    seed = rank_seed(w.seed, rank)
    rng = np.random.Generator(np.random.PCG64(seed))
    kk = args.k if args.k > 0 else w.k
    past = np.full(w.B, w.n, np.int32)
    cand = np.full(w.B, kk, np.int32)
    H, D, L, S, n_cap = w.H, w.D, w.L, w.S, w.n_cap
    if args.layers > 0:
        L = args.layers        # smaller pool and fewer layer calls per step (profiler captures)
    slots = rng.permutation(S)[: w.B].astype(np.int32)

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    pool_k = torch.full((L, S, H, n_cap, D), 0x7FC0, dtype=torch.int16, device=device).view(torch.bfloat16)
    pool_v = torch.full((L, S, H, n_cap, D), 0x7FC0, dtype=torch.int16, device=device).view(torch.bfloat16)
    for layer in range(L):                     # cached rows of every request, every layer
        ks, vs = synth.pool_rows(rng, past, H, D)
        for r in range(w.B):
            pool_k[layer, int(slots[r]), :, : w.n] = dev_bf16(ks[r])
            pool_v[layer, int(slots[r]), :, : w.n] = dev_bf16(vs[r])
    Tc = int(cand.sum())
    qs, kc, vc = [], [], []
    for layer in range(L):                     # fresh candidate q/k/v per layer
        qs.append(dev_bf16(synth.normal_bf16(rng, (Tc, H, D))))
        kc.append(dev_bf16(synth.normal_bf16(rng, (Tc, H, D))))
        vc.append(dev_bf16(synth.normal_bf16(rng, (Tc, H, D))))
    cu = torch.from_numpy(synth.cu_from_lens(cand)).to(device)
    pl = torch.from_numpy(past).to(device)
    sl = torch.from_numpy(slots).to(device)
    out = [torch.empty((Tc, H, D), dtype=torch.bfloat16, device=device) for _ in range(L)]
    pool_scales = None
    if args.pool == "e4m3":
        # the same rows as E4M3 codes of x / 2^-6 (a bfloat16-valued scale: N(0,1) rows up to 7)
        pool_scales = (2.0 ** -6, 2.0 ** -6)
        k8 = torch.empty((L, S, H, n_cap, D), dtype=torch.float8_e4m3fn, device=device)
        v8 = torch.empty_like(k8)
        for layer in range(L):
            k8[layer] = (pool_k[layer].float() / pool_scales[0]).to(torch.float8_e4m3fn)
            v8[layer] = (pool_v[layer].float() / pool_scales[1]).to(torch.float8_e4m3fn)
        pool_k, pool_v = k8, v8
        torch.cuda.empty_cache()
    ws_bytes = ub.rank_decode_pool_workspace_size(pool_k, pool_v, w.B, H, kk, Tc, pool_scales=pool_scales)
    ws = torch.empty(ws_bytes // 4 + 4, dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)

    def layers(s):
        for layer in range(L):
            ub.rank_decode_attn(qs[layer], kc[layer], vc[layer], cu, sl, pl, pool_k, pool_v, layer, kk,
                                out=out[layer], out_fp32=False, workspace=ws, dev_status=status, stream=s,
                                pool_scales=pool_scales)

    graph = None

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            layers(stream)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if args.graph:
        # the L layer calls of a step as one CUDA graph (every call is asynchronous, allocates
        # nothing and syncs nothing, and the first calls above did the one-time set-up)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layers(torch.cuda.current_stream(device))
        torch.cuda.synchronize(device)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(device)
    clk = clocks.stop() if clocks else None
    if int(status.item()) != 0:
        raise RuntimeError("device status %s" % ub.status_string(int(status.item())))
    ms_step = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    peaks = load_peaks()
    flops = decode_flops(past, cand, H, D) * L
    nbytes = decode_bytes(past, cand, H, D, 2, 1 if pool_scales else 2) * L
    tflops = flops / (ms_step * 1e-3) / 1e12
    gbs = nbytes / (ms_step * 1e-3) / 1e9
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    roof = ({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": gbs / peaks["hbm_gbs"]} if bound == "hbm" else
            {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": tflops / peaks["bf16_tflops"]})
    # the library sends requests of at most 64 candidates (one query head per kv head) to the small-k
    # kernel; over an E4M3 pool it reads the codes in place up to 32 columns at D=64 (64 at D=128)
    n_pad = 16 if kk <= 16 else 32 if kk <= 32 else 64
    if kk <= 64 and D in (64, 128):
        kernel = "decode_smallk_kernel<%d,%d>" % (D, n_pad)
        if pool_scales and (n_pad <= 32 or D == 128):
            kernel = "decode_smallk_kernel<%d,%d,e4m3>" % (D, n_pad)
        elif pool_scales:
            kernel = "kvpool_dequant_kernel + " + kernel
    else:
        kernel = ("kvpool_dequant_kernel + " if pool_scales else "") + "attn_fwd_kernel<%d,decode>" % D
    roof.update({"kernel": kernel, "traffic": None, "peak_source": "%s (burst for tensor)" % peaks["source"]})
    return {
        "metric": METRIC, "value": float(cand.sum()) * L / (ms_step * 1e-3), "unit": "candidate tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name if args.layers <= 0 else "%s[layers=%d]" % (w.name, L),
                   "requests": w.B, "k": kk, "n": w.n, "H": H, "D": D,
                   "pool": [L, S, H, n_cap, D], "layers_per_step": L, "split_n": ws_bytes > 256,
                   "pool_dtype": args.pool, "pool_scales": pool_scales,
                   "cuda_graph": bool(args.graph),
                   "l2": "pool slots read per step exceed L2 (no flush)"},
        "phases": {"decode_tflops": tflops, "decode_gbs": gbs, "decode_frac_hbm": gbs / peaks["hbm_gbs"],
                   "decode_frac_tensor": tflops / peaks["bf16_tflops"],
                   "roof_time_ms": 1e3 * max(t_hbm, t_tc)},
        "roofline": roof,
        "gpu_launches": args.steps * L * ((2 if (ws_bytes > 256 and kk > 128) else 1) +
                                          (1 if kernel.startswith("kvpool_dequant") else 0)),
        "clocks": clk,
    }


def run_backward_only(args, rank, world, device, dist):
    """Gradients of the masked prefill: one forward for out and lse, then the timed backward calls."""
    import torch
    from kv_cache_reuse_falcon_b200 import binding as ub

    w = synth.workload(args.workload)
    rng = np.random.Generator(np.random.PCG64(rank_seed(w.seed, rank)))
    past, cand = w.lengths(rng)
    cu_h = synth.cu_from_lens(past + cand)
    T = int(cu_h[-1])

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    q, k, v, g = (dev_bf16(synth.normal_bf16(rng, (T, w.H, w.D))) for _ in range(4))
    cu = torch.from_numpy(cu_h).to(device)
    pl = torch.from_numpy(past).to(device)
    max_len = int((past + cand).max())
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    lse = torch.empty((T, w.H), dtype=torch.float32, device=device)
    o = ub.masked_prefill_attn(q, k, v, cu, pl, max_len, out_fp32=False, lse=lse, dev_status=status)
    grads = [torch.empty((T, w.H, w.D), dtype=torch.float32, device=device) for _ in range(3)]
    ws = torch.empty(ub.masked_prefill_bwd_workspace_size(T, w.H) // 4 + 4, dtype=torch.float32, device=device)

    def step():
        ub.masked_prefill_bwd(q, k, v, o, g, lse, cu, pl, max_len, dq=grads[0], dk=grads[1], dv=grads[2],
                              workspace=ws, dev_status=status, stream=stream)

    for _ in range(args.warmup):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    for i in range(args.steps):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop() if clocks else None
    if int(status.item()) != 0:
        raise RuntimeError("device status %s" % ub.status_string(int(status.item())))
    ms_step = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    peaks = load_peaks()
    flops = 2.5 * prefill_flops(past, cand, w.H, w.D)
    e = roof_entry(ms_step, flops, 5 * T * w.H * w.D * 2 + 3 * T * w.H * w.D * 4 + 2 * T * w.H * 4, peaks,
                   "bwd_prep_kernel<%d> + bwd_kv_kernel<%d>" % (w.D, w.D))
    return {
        "metric": METRIC, "value": float(T) / (ms_step * 1e-3), "unit": "tokens/s (backward)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "n": w.n, "k": w.k, "H": w.H, "D": w.D, "tokens": T,
                   "l2": "inputs larger than L2 (no flush)"},
        "roofline": {"bound": e["bound"], "achieved": e["tflops"] if e["bound"] == "tensor" else e["gbs"],
                     "peak": peaks["bf16_tflops"] if e["bound"] == "tensor" else peaks["hbm_gbs"],
                     "unit": "TFLOP/s" if e["bound"] == "tensor" else "GB/s", "frac": e["frac_roof"],
                     "kernel": e["kernel"], "traffic": None, "peak_source": peaks["source"]},
        "gpu_launches": args.steps * 2, "clocks": clk,
    }


def run_reference(args, rank, world):
    """The oracle (fp64 CPU) timed on the host cores, a bounded sample of the same workload per step."""
    if rank != 0:
        return None
    w = synth.workload(args.workload)
    name = w.name
    _, batch, _, _ = make_workload(name, w.seed)
    for _ in range(args.warmup):
        cpu_oracle_sample(batch, budget_s=0.5, max_segments=1, seed=99)
    vals = []
    per_step = max(2.0, min(20.0, 150.0 / max(args.steps, 1)))
    sample = None
    for i in range(args.steps):
        r = cpu_oracle_sample(batch, budget_s=per_step, seed=i)
        vals.append(r["value"])
        sample = r
    value = float(statistics.median(vals))
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "candidate tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": None,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": name if not args.users else "%s[users=%d]" % (name, args.users),
                   "users_per_gpu": batch.B, "H": batch.H, "D": batch.D},
        "cpu_baseline": {"value": value, "unit": "candidate tokens/s", "cores": sample["cores"], "kind": "oracle",
                         "sample": sample["sample"]},
        "e2e": {"value": value, "unit": "candidate tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def relaunch_command(argv, nproc, port=None):
    """torchrun command that runs this script once per GPU (rendezvous on 127.0.0.1)."""
    if port is None:
        import socket
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(nproc),
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--users", type=int, default=0, help="smaller case: this many users (profiling)")
    ap.add_argument("--k", type=int, default=0, help="decode workloads: candidates per request")
    ap.add_argument("--pool", default="bf16", choices=["bf16", "e4m3"],
                    help="decode workloads: the pool's element type (E4M3 codes with scale 2^-6)")
    ap.add_argument("--layers", type=int, default=0,
                    help="decode workloads: pool layers and layer calls per step (smaller case)")
    ap.add_argument("--no-sweep", action="store_true", help="headline workload only (no per-config sweep)")
    ap.add_argument("--graph", action="store_true",
                    help="decode workloads: replay each step's layer calls as one CUDA graph")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        if args.impl == "reference":
            args.gpus = 1   # the oracle runs on rank 0's host cores only
        else:
            # one process per GPU: start the ranks with torch's launcher; rank 0 prints the line
            return subprocess.call(relaunch_command(argv if argv is not None else sys.argv[1:], args.gpus))
    world = int(world_env or "1")
    if args.impl != "reference" and world != args.gpus:
        ap.error("--gpus %d but the launcher started %d ranks (WORLD_SIZE)" % (args.gpus, world))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
        dist = tdist
    try:
        if synth.workload(args.workload).kind == "decode":
            res = run_decode_only(args, rank, world, device, dist)
        elif synth.workload(args.workload).kind == "backward":
            res = run_backward_only(args, rank, world, device, dist)
        else:
            res = run_ours(args, rank, world, device, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
