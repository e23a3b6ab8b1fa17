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
from kv_cache_reuse_falcon_b200.shard import rank_seed, segment_cost  # noqa: E402

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


def decode_bytes(past, cand, H, D, out_bytes):
    """Algorithmic bytes: pool K/V rows read once + candidate q/k/v read + output written."""
    p = np.asarray(past, dtype=np.float64).sum()
    k = np.asarray(cand, dtype=np.float64).sum()
    return float(2 * p * H * D * 2 + 3 * k * H * D * 2 + k * H * D * out_bytes)


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
    # kernel_source_key() of csrc/attn_sm100.cuh, H, D: bytes per token
    ("03012fff8e2df70c", 8, 128): (431.669760e6 + 123.166208e6) / 70236,
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
        if ev is not None:
            ev[0].record(stream)
        ub.kvpool_write(pool_k, pool_v, layer, k, v, cu, pl, sl, max_past, dev_status=status, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        ub.masked_prefill_attn(q, k, v, cu, pl, max_seqlen, out=out_p, out_fp32=False, workspace=ws_pre,
                               dev_status=status, stream=stream)
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
    t_pool = [e[0].elapsed_time(e[1]) for e in evs]
    t_pre = [e[1].elapsed_time(e[2]) for e in evs]
    t_dec = [e[2].elapsed_time(e[3]) for e in evs]
    if int(status.item()) != 0:
        raise RuntimeError("device status %s in the timed region" % ub.status_string(int(status.item())))

    # ------------------------------------------------------ end to end (host buffers)
    hq = torch.from_numpy(batch.q.view(np.int16)).pin_memory()
    hk = torch.from_numpy(batch.k.view(np.int16)).pin_memory()
    hv = torch.from_numpy(batch.v.view(np.int16)).pin_memory()
    hqc = torch.from_numpy(np.ascontiguousarray(batch.q[cidx]).view(np.int16)).pin_memory()
    hkc = torch.from_numpy(np.ascontiguousarray(batch.k[cidx]).view(np.int16)).pin_memory()
    hvc = torch.from_numpy(np.ascontiguousarray(batch.v[cidx]).view(np.int16)).pin_memory()
    hcu = torch.from_numpy(batch.cu_seqlens.astype(np.int32)).pin_memory()
    hpl = torch.from_numpy(past.astype(np.int32)).pin_memory()
    hsl = torch.from_numpy(batch.slot_ids.astype(np.int32)).pin_memory()
    hcuc = torch.from_numpy(synth.cu_from_lens(cand)).pin_memory()
    hout = torch.empty((Tc, H, D), dtype=torch.bfloat16).pin_memory()
    h2d = [(hq, q.view(torch.int16)), (hk, k.view(torch.int16)), (hv, v.view(torch.int16)),
           (hqc, qc.view(torch.int16)), (hkc, kc.view(torch.int16)), (hvc, vc.view(torch.int16)),
           (hcu, cu), (hpl, pl), (hsl, sl), (hcuc, cu_c)]
    h2d_bytes = sum(h.numel() * h.element_size() for h, _ in h2d)
    d2h_bytes = hout.numel() * hout.element_size()
    e2e_steps = max(1, min(args.steps, 3))
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for h, d in h2d:
            d.copy_(h, non_blocking=True)
        step()
        hout.copy_(out_d, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    # ---------------------------------------------------------- max over ranks
    ms_step = elapsed_ms / args.steps
    pre_ms = sum(t_pre) / len(t_pre)
    dec_ms = sum(t_dec) / len(t_dec)
    pool_ms = sum(t_pool) / len(t_pool)
    cand_total = float(cand.sum())
    if dist is not None:
        import torch.distributed as tdist
        t = torch.tensor([ms_step, e2e_ms, pre_ms, dec_ms, pool_ms], dtype=torch.float64, device=device)
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        ms_step, e2e_ms, pre_ms, dec_ms, pool_ms = [float(x) for x in t.tolist()]
        c = torch.tensor([cand_total], dtype=torch.float64, device=device)
        tdist.all_reduce(c, op=tdist.ReduceOp.SUM)
        cand_total = float(c.item())

    peaks = load_peaks()
    pf = prefill_flops(past, cand, H, D)
    df = decode_flops(past, cand, H, D)
    db = decode_bytes(past, cand, H, D, 2)
    pwb = pool_write_bytes(past, H, D)
    pre_tflops = pf / (pre_ms * 1e-3) / 1e12
    dec_tflops = df / (dec_ms * 1e-3) / 1e12
    dec_gbs = db / (dec_ms * 1e-3) / 1e9
    pool_gbs = pwb / (pool_ms * 1e-3) / 1e9
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
        "phases": {"pool_write_ms": pool_ms, "prefill_ms": pre_ms, "decode_ms": dec_ms,
                   "prefill_tflops": pre_tflops, "decode_tflops": dec_tflops, "decode_gbs": dec_gbs,
                   "pool_write_gbs": pool_gbs,
                   "prefill_frac_tensor": pre_tflops / peak,
                   "prefill_frac_tensor_sustained": pre_tflops / peaks["bf16_tflops_sustained"],
                   "decode_frac_hbm": dec_gbs / peaks["hbm_gbs"],
                   "pool_write_frac_hbm": pool_gbs / peaks["hbm_gbs"]},
        "roofline": {"kernel": "attn_fwd_kernel<128,prefill>", "bound": "tensor", "achieved": pre_tflops,
                     "peak": peak, "unit": "TFLOP/s", "frac": pre_tflops / peak,
                     "traffic": prefill_traffic(T, H, D),
                     "traffic_note": "ncu DRAM bytes per token of a 24-user capture, scaled by tokens",
                     "peak_source": "%s bf16_tflops (burst)" % peaks["source"],
                     "work_per_launch": "4*D*H*sum_b[n_b(n_b+1)/2 + k_b(n_b+1)] = %.4g FLOP" % pf},
        "e2e": {"value": cand_total / (e2e_ms * 1e-3), "unit": "candidate tokens/s",
                "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes),
                "steps": e2e_steps},
        "gpu_launches": args.steps * (3 + (1 if decode_split else 0)),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_oracle_sample(batch, budget_s=args.cpu_budget)
    return result


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
    ws_bytes = ub.rank_decode_workspace_size(w.B, H, D, kk, Tc, n_cap)
    ws = torch.empty(ws_bytes // 4 + 4, dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)

    def layers(s):
        for layer in range(L):
            ub.rank_decode_attn(qs[layer], kc[layer], vc[layer], cu, sl, pl, pool_k, pool_v, layer, kk,
                                out=out[layer], out_fp32=False, workspace=ws, dev_status=status, stream=s)

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
    nbytes = decode_bytes(past, cand, H, D, 2) * L
    tflops = flops / (ms_step * 1e-3) / 1e12
    gbs = nbytes / (ms_step * 1e-3) / 1e9
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    roof = ({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": gbs / peaks["hbm_gbs"]} if bound == "hbm" else
            {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": tflops / peaks["bf16_tflops"]})
    roof.update({"kernel": "attn_fwd_kernel<%d,decode>" % D, "traffic": None,
                 "peak_source": "%s (burst for tensor)" % peaks["source"]})
    return {
        "metric": METRIC, "value": float(cand.sum()) * L / (ms_step * 1e-3), "unit": "candidate tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name if args.layers <= 0 else "%s[layers=%d]" % (w.name, L),
                   "requests": w.B, "k": kk, "n": w.n, "H": H, "D": D,
                   "pool": [L, S, H, n_cap, D], "layers_per_step": L, "split_n": ws_bytes > 256,
                   "cuda_graph": bool(args.graph),
                   "l2": "pool slots read per step exceed L2 (no flush)"},
        "phases": {"decode_tflops": tflops, "decode_gbs": gbs, "decode_frac_hbm": gbs / peaks["hbm_gbs"],
                   "decode_frac_tensor": tflops / peaks["bf16_tflops"],
                   "roof_time_ms": 1e3 * max(t_hbm, t_tc)},
        "roofline": roof, "gpu_launches": args.steps * L * (2 if ws_bytes > 256 else 1), "clocks": clk,
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
    ap.add_argument("--layers", type=int, default=0,
                    help="decode workloads: pool layers and layer calls per step (smaller case)")
    ap.add_argument("--graph", action="store_true",
                    help="decode workloads: replay each step's layer calls as one CUDA graph")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
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
