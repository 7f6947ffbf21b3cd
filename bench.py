"""Benchmark of the Prism block-sparse attention path (one prefill attention layer).

A step is one pass of the whole path over one layer of synthetic input already
resident in HBM: sfa_block_scores (RoPE + dual-band pooling + energy
temperature + block scores), sfa_select, sfa_block_sparse_attn.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Every rank runs an independent
replica of the layer (the path has no exchange step between layers' units;
"scaling": "weak").  Rank 0 prints one JSON line.

value  = attention FLOPs over the kept blocks (causal diagonal counted half),
         summed over ranks, / the slowest rank's device time for K steps -> TFLOP/s.
e2e    = the same metric through sfa.HostPipeline from pinned host tensors:
         H2D of Q, K, V and D2H of O for every timed step, on two copy streams
         overlapping the path of the neighbouring steps (double-buffered).
--impl reference times the CPU oracle (the slow fp64 restatement) on a
bounded sample of the same workload (see cpu_baseline.sample).

--workload fasa-decode-* runs the decode step instead (one query token per
sequence against a KV cache: compact-key append for the new position, token
importance + top-k, focused attention): value = decode tokens/s (sequences x
steps / time), roofline of the selection on the compact-key stream (HBM).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_dual_b200 import workloads as wl  # noqa: E402
from block_sparse_long_dual_b200.synthetic import make_inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 5  # rope_pool_energy, band_temperature, block_score_softmax, select, attention (4 when fused)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=wl.LLAMA_128K.name, choices=sorted(wl.ALL) + sorted(wl.DECODE))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--fused", action="store_true",
                    help="estimate and selection in one call (sfa_block_scores_select; probabilities not stored)")
    ap.add_argument("--rope-on-load", action="store_true",
                    help="the attention rotates Q as it loads it (sfa_block_sparse_attn_rope; Q_rot not stored)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attention_flops(counts: np.ndarray, block: int, d: int) -> float:
    """4*d*(block^2 per off-diagonal kept block + block(block+1)/2 per diagonal block), summed."""
    n = counts.astype(np.float64)
    diag = (n > 0).astype(np.float64)  # the diagonal block is always in the selection
    return float(4.0 * d * (block * block * (n - diag) + block * (block + 1) / 2.0 * diag).sum())


def scoring_bytes(w: wl.Workload, store_probs: bool = True, store_q_rot: bool = True) -> float:
    """Algorithmic HBM bytes of sfa_block_scores: read Q, K; write Q_r (unless the attention
    rotates Q on load), K_r; read the cos/sin table once; write the float64 block means; write
    probs [B, Hq, nb, nb] (unless the selection is fused and the probabilities are not stored)."""
    e = 2 if w.dtype == "bf16" else 4
    qk = w.batch * (w.heads_q + w.heads_kv) * w.seq_len * w.head_dim * e
    k_only = w.batch * w.heads_kv * w.seq_len * w.head_dim * e
    table = 2 * w.seq_len * (w.head_dim // 2) * 4
    means = w.batch * (w.heads_q + w.heads_kv) * w.nb * w.head_dim * 8
    probs = w.batch * w.heads_q * w.nb * w.nb * 4 if store_probs else 0
    return float(qk + (qk if store_q_rot else k_only) + table + means + probs)


def select_bytes(w: wl.Workload, kmax: int, read_probs: bool = True) -> float:
    """Read the causal triangle of probs (unless the selection is fused), write counts and idx."""
    tri = w.batch * w.heads_q * w.nb * (w.nb + 1) / 2 * 4 if read_probs else 0
    return float(tri + w.batch * w.heads_q * w.nb * (1 + kmax) * 4)


def traffic_record(kernel_file: str):
    """ncu DRAM bytes per launch of the attention kernel, if captured for the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for fn in rec.get("sources", []):
        with open(os.path.join(ROOT, fn), "rb") as f:
            h.update(f.read())
    if rec.get("sha256") != h.hexdigest():
        return None
    return rec


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period, self.index = period_s, index
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        names = {
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def oracle_head_sample(w: wl.Workload, Q, K, V, h: int = 0, attn_blocks: int | None = None):
    """Time the CPU oracle on one (batch 0, Q head h) unit of the workload.

    Runs the estimate, the selection of every row and exact attention over
    ``attn_blocks`` evenly spaced query blocks (all when None); the attention
    time is scaled to all query blocks of the head.  Returns (TFLOP/s, seconds, sample text)."""
    from oracle import prism_oracle as po
    g = h // w.group
    Qh = Q[0:1, h:h + 1].to(torch.float64).numpy()
    Kh = K[0:1, g:g + 1].to(torch.float64).numpy()
    Vh = V[0:1, g:g + 1].to(torch.float64).numpy()
    mass = None if w.mass is None else float(np.float32(w.mass))
    t0 = time.perf_counter()
    cos, sin = po.rope_tables(w.rope_base, w.seq_len, w.head_dim)
    sc = po.prism_scores(Qh, Kh, w.block, w.band_split, w.flags, (cos, sin))
    sel = po.select_blocks(sc.probs, w.flags, k=w.k, mass=mass)
    qa = po.round_to_dtype(sc.q_rot, w.dtype)
    ka = po.round_to_dtype(sc.k_rot, w.dtype)
    t1 = time.perf_counter()
    nb = w.nb
    rows = list(range(nb)) if attn_blocks is None or attn_blocks >= nb else \
        sorted(set(np.linspace(0, nb - 1, attn_blocks).astype(int).tolist()))
    keep = set(rows)
    kept = [[[sel[0][0][i].kept if i in keep else np.zeros(0, np.int64) for i in range(nb)]]]
    po.sparse_attention(qa, ka, Vh, kept, w.block)
    t2 = time.perf_counter()
    counts = np.array([sel[0][0][i].kept.size for i in range(nb)])
    flops = attention_flops(counts, w.block, w.head_dim)
    secs = (t1 - t0) + (t2 - t1) * nb / len(rows)
    text = (f"batch 0, Q head {h} of {w.heads_q}: RoPE tables, estimate and selection over the full "
            f"{w.seq_len}-token head, exact attention on {len(rows)} of {nb} query blocks"
            + ("" if len(rows) == nb else f" (attention time scaled by {nb}/{len(rows)})"))
    return flops / secs / 1e12, secs, text


def layer_config(w: wl.Workload, world: int) -> dict:
    """The config keys both arms report for a prefill workload."""
    return {"workload": w.name,
            "layer": f"B={w.batch} Hq={w.heads_q} Hkv={w.heads_kv} L={w.seq_len} d={w.head_dim} "
                     f"block={w.block} rope_base={w.rope_base:g} band_split={w.band_split}",
            "budget": (f"top-{w.k} + diagonal" if w.k is not None else f"mass {w.mass}"),
            "parallelism": f"replicas x{world}"}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), for the oracle timings."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i["num_threads"] for i in threadpool_info()] or [1])
    except Exception:
        return None


DECODE_METRIC = "decode tokens/s (one query token per sequence per step, TIP + top-k + focused attention)"


def decode_bytes(w: wl.DecodeWorkload):
    """Algorithmic HBM bytes of one decode step: (selection) the compact keys [B, Hkv, L, 2 nfc]
    and q; (attention) the k kept K and V rows of every (b, h), q, o; (append) one compact row per
    (b, KV head).  Returns (selection bytes, attention bytes, total)."""
    sel = w.batch * w.heads_kv * w.seq_len * 2 * w.nfc * 2 + w.batch * w.heads_q * w.head_dim * 2
    att = w.batch * w.heads_q * (w.k * 2 * w.head_dim * 2 + 2 * w.head_dim * 2 + w.k * 4)
    app = w.batch * w.heads_kv * (w.head_dim * 2 + 2 * w.nfc * 2)
    return float(sel), float(att), float(sel + att + app)


def oracle_decode_sample(w: wl.DecodeWorkload, q, K, V, fc, b=0, h=0):
    """Time the oracle's decode step on one (b, h) row; returns (tokens/s, seconds, sample text)."""
    from oracle import fasa_oracle as fo
    g = h // w.group
    qn = q[b:b + 1, h:h + 1].to(torch.float64).numpy()
    Kn = K[b:b + 1, g:g + 1].to(torch.float64).numpy()
    Vn = V[b:b + 1, g:g + 1].to(torch.float64).numpy()
    t0 = time.perf_counter()
    fo.decode_step(qn, Kn, Vn, fc[g:g + 1], w.k)
    secs = time.perf_counter() - t0
    # a step is batch x heads_q such rows for batch tokens
    value = w.batch / (secs * w.batch * w.heads_q)
    text = (f"one (sequence, Q head) row of {w.batch} x {w.heads_q}: float64 importance over the {w.seq_len}-token "
            f"cache, top-{w.k}, float64 attention; scaled to the full step")
    return value, secs, text


def run_decode(args, w: wl.DecodeWorkload, rank, world):
    from block_sparse_long_dual_b200 import sfa
    from block_sparse_long_dual_b200.synthetic import make_decode_inputs
    if args.impl == "reference":
        if rank != 0:
            return
        q, K, V, fc = make_decode_inputs(w.scaled(batch=1), seed=0)
        per = []
        text = ""
        for s_ in range(args.warmup + args.steps):
            v, secs, text = oracle_decode_sample(w.scaled(batch=1), q, K, V, fc, 0, s_ % w.heads_q)
            if s_ >= args.warmup:
                per.append((v, secs))
        value = float(np.mean([v for v, _ in per]))
        line = {"metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": float(np.mean([s for _, s in per])) * 1e3 * w.heads_q,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "impl": "reference",
                "config": {"workload": w.name},
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads() or
                                 len(os.sched_getaffinity(0)), "kind": "oracle", "sample": text, "cpu_model": cpu_model()},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    q, K, V, fc = make_decode_inputs(w, seed=rank)
    m = sfa.FasaDecode(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len,
                       head_dim=w.head_dim, fc=fc, k=w.k, device=dev)
    qd, Kd, Vd = q.to(dev), K.to(dev), V.to(dev)
    m.refresh_keys(Kd)
    stream = torch.cuda.current_stream(dev)

    def step():
        m.refresh_keys(Kd, pos0=w.seq_len - 1, npos=1)   # compact row of the newest position
        m.select(qd)
        m.attend(qd, Kd, Vd)

    for _ in range(max(args.warmup, 3)):
        step()
        m.step(qd, Kd, Vd, w.seq_len - 1)   # the same step as one CUDA graph (captured once)
    torch.cuda.synchronize(dev)
    if int(m.status.item()) != 0:
        raise RuntimeError(f"device status {int(m.status.item())}")
    # stage times: each stage captured as a CUDA graph of its own and replayed back to back, so
    # that host launch costs do not show up as device time
    def graph_ms(fn, reps):
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(reps):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        return g0.elapsed_time(g1) / reps

    # at least 500 step replays (~50 ms at 128K x 4), so that the clock sampler sees the timed region
    K_ = max(args.steps, 500)
    t_app = graph_ms(lambda: m.refresh_keys(Kd, pos0=w.seq_len - 1, npos=1), K_)
    t_sel = graph_ms(lambda: m.select(qd), K_)
    t_att = graph_ms(lambda: m.attend(qd, Kd, Vd), K_)
    # the timed steps: graph replays back to back
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for s_ in range(K_):
            m.step(qd, Kd, Vd, w.seq_len - 1)
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    total_ms = start.elapsed_time(stop)

    # e2e: pinned host q in, o out, through the public API
    qh = q.pin_memory()
    oh = torch.empty(m.o.shape, dtype=m.o.dtype).pin_memory()
    qdev = torch.empty_like(qd)

    def host_step():
        qdev.copy_(qh, non_blocking=True)
        m.step(qdev, Kd, Vd, w.seq_len - 1)
        oh.copy_(m.o, non_blocking=True)

    host_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K_):
        host_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    vals = torch.tensor([total_ms, e2e_ms, t_sel, t_att, t_app], dtype=torch.float64, device=dev)
    if dist:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    total_ms, e2e_ms, t_sel, t_att, t_app = vals.tolist()
    if rank == 0:
        pk, pk_src = peaks()
        sel_b, att_b, all_b = decode_bytes(w)
        achieved = sel_b / (t_sel * 1e-3) / 1e9
        line = {
            "metric": DECODE_METRIC, "value": w.batch * world * K_ / (total_ms * 1e-3), "unit": "tokens/s",
            "n_gpus": world, "steps": K_, "warmup": max(args.warmup, 3), "ms_per_step": total_ms / K_,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name,
                       "cache": f"B={w.batch} Hq={w.heads_q} Hkv={w.heads_kv} L={w.seq_len} d={w.head_dim}",
                       "dominant_pairs": w.nfc, "k": w.k, "parallelism": f"replicas x{world}",
                       "launch": "each step one CUDA graph of its four kernels (FasaDecode.step)",
                       "l2": "compact keys 201 MB, K/V cache 2.1 GB per GPU (larger than L2); no flush"},
            "stages_us": {"append": t_app * 1e3, "select": t_sel * 1e3, "attention": t_att * 1e3},
            "roofline": {"kernel": "tip_chunk + tip_merge (sfa_decode_select)", "bound": "hbm",
                         "achieved": achieved, "peak": float(pk["hbm_gbs"]), "unit": "GB/s",
                         "frac": achieved / float(pk["hbm_gbs"]), "peak_source": f"{pk_src} HBM copy",
                         "traffic": None, "bytes_per_launch": sel_b},
            "step_bytes": all_b,
            "e2e": {"value": w.batch * K_ / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": qh.numel() * qh.element_size(),
                    "d2h_bytes_per_step": oh.numel() * oh.element_size()},
            "gpu_launches": 4 * K_,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            v, secs, text = oracle_decode_sample(w, q, K, V, fc)
            line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": blas_threads() or
                                    len(os.sched_getaffinity(0)), "kind": "oracle", "sample": text,
                                    "seconds": secs, "cpu_model": cpu_model()}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, w, rank, world):
    """The reference arm: the CPU oracle as it stands, on host cores, bounded sample per step."""
    if rank != 0:
        return
    Q, K, V = make_inputs(w.scaled(batch=1), seed=0)
    per_step = []
    blocks = max(4, min(64, w.nb // 16))
    text = ""
    wall = []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        v, secs, text = oracle_head_sample(w, Q, K, V, h=s % w.heads_q, attn_blocks=blocks)
        if s >= args.warmup:
            per_step.append((v, secs))
            wall.append(time.perf_counter() - t0)
    value = float(np.mean([v for v, _ in per_step]))
    ms = float(np.mean([s for _, s in per_step]) * 1e3)
    cores = len(os.sched_getaffinity(0))
    line = {"metric": "prefill attention effective TFLOP/s over kept blocks (whole path)", "value": value,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference", "extrapolated": True,
            "measured_ms_per_step": float(np.mean(wall)) * 1e3,
            "config": layer_config(w, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads() or cores,
                             "kind": "oracle", "sample": text, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in wl.DECODE:
        run_decode(args, wl.DECODE[args.workload], rank, world)
        return
    w = wl.ALL[args.workload]
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    from block_sparse_long_dual_b200 import sfa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    Q, K, V = make_inputs(w, seed=rank)
    model = sfa.PrismAttention(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len,
                               head_dim=w.head_dim, dtype=w.dtype, block=w.block, rope_base=w.rope_base,
                               band_split=w.band_split, k=w.k, mass=w.mass, flags=w.flags, device=dev,
                               fused=args.fused, rope_on_load=args.rope_on_load)
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        model(Qd, Kd, Vd)
    torch.cuda.synchronize(dev)
    if int(model.status.item()) != 0:
        raise RuntimeError(f"device status {int(model.status.item())}")

    K_ = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for s in range(K_):
            ev[s][0].record(stream)
            if args.fused:
                model.scores_select(Qd, Kd)
            else:
                model.scores(Qd, Kd)
            ev[s][1].record(stream)
            if not args.fused:
                model.select()
            ev[s][2].record(stream)
            model.attend(Vd, Qd)
            ev[s][3].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    total_ms = start.elapsed_time(stop)
    t_scores = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K_)]
    t_select = [ev[s][1].elapsed_time(ev[s][2]) for s in range(K_)]
    t_attn = [ev[s][2].elapsed_time(ev[s][3]) for s in range(K_)]

    counts = model.counts.cpu().numpy()
    flops_step = attention_flops(counts, w.block, w.head_dim)
    kept_frac = float(counts.sum()) / (w.batch * w.heads_q * w.nb * (w.nb + 1) / 2)

    # e2e: the public API from pinned host buffers, every step's copies inside the timed region
    # (uploads and downloads on their own streams, overlapping the neighbouring steps' path)
    e2e_steps = args.e2e_steps or K_
    Qh, Kh, Vh = (t.pin_memory() for t in (Q, K, V))
    Oh = [torch.empty(model.O.shape, dtype=model.O.dtype).pin_memory() for _ in range(2)]
    pipe = sfa.HostPipeline(model, Qd, Kd, Vd)
    for i in range(2):
        pipe.submit(Qh, Kh, Vh, Oh[i])
    pipe.drain()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    pipe.up.wait_stream(stream)
    pipe.down.wait_stream(stream)
    for i in range(e2e_steps):
        pipe.submit(Qh, Kh, Vh, Oh[i % 2])
    pipe.drain(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if int(model.status.item()) != 0:
        raise RuntimeError(f"device status {int(model.status.item())}")
    h2d = sum(t.numel() * t.element_size() for t in (Qh, Kh, Vh))
    d2h = Oh[0].numel() * Oh[0].element_size()
    # The host links alone (no layer): the same uploads, then uploads and downloads together.
    link_ms = []
    for both in (False, True):
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        l0.record(stream)
        pipe.up.wait_stream(stream)
        pipe.down.wait_stream(stream)
        for i in range(3):
            with torch.cuda.stream(pipe.up):
                for d, hst in zip(pipe.dev_in[i % 2], (Qh, Kh, Vh)):
                    d.copy_(hst, non_blocking=True)
            if both:
                with torch.cuda.stream(pipe.down):
                    Oh[i % 2].copy_(pipe.dev_out[(i + 1) % 2], non_blocking=True)
        stream.wait_stream(pipe.up)
        stream.wait_stream(pipe.down)
        l1.record(stream)
        torch.cuda.synchronize(dev)
        link_ms.append(l0.elapsed_time(l1) / 3)

    vals = torch.tensor([total_ms, e2e_ms, float(np.mean(t_attn)), float(np.mean(t_scores)),
                         float(np.mean(t_select))], dtype=torch.float64, device=dev)
    fl = torch.tensor([flops_step], dtype=torch.float64, device=dev)
    if dist:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(fl, op=dist.ReduceOp.SUM)
    total_ms, e2e_ms, attn_ms, scores_ms, select_ms = vals.tolist()
    flops_all = fl.item()

    if rank == 0:
        pk, pk_src = peaks()
        value = flops_all * K_ / (total_ms * 1e-3) / 1e12
        e2e_value = flops_all * e2e_steps / (e2e_ms * 1e-3) / 1e12
        achieved = flops_step / (attn_ms * 1e-3) / 1e12
        peak = float(pk["bf16_tflops"])
        tr = traffic_record("block_sparse_long_dual_b200/csrc/attn_tc.cu")
        sb = scoring_bytes(w, not args.fused, not args.rope_on_load)
        selb = select_bytes(w, model.kmax, not args.fused)
        line = {
            "metric": "prefill attention effective TFLOP/s over kept blocks (whole path)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K_, "warmup": args.warmup,
            "ms_per_step": total_ms / K_, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {**layer_config(w, world), "kept_fraction": round(kept_frac, 5),
                       "estimate": ("fused with the selection (sfa_block_scores_select, probabilities not stored)"
                                    if args.fused else "sfa_block_scores then sfa_select"),
                       "attention": ("RoPE on load (sfa_block_sparse_attn_rope: Q rotated in the attention kernel, "
                                     "Q_rot not stored)" if args.rope_on_load else "sfa_block_sparse_attn on Q_rot"),
                       "l2": "inputs larger than L2 (Q 1.07 GB, K 0.27 GB, V 0.27 GB at 128K); no flush"},
            "stages_ms": {"block_scores": scores_ms, "select": select_ms, "attention": attn_ms},
            "scoring": {"bytes": sb + selb, "GB_s": (sb + selb) / ((scores_ms + select_ms) * 1e-3) / 1e9,
                        "frac_hbm": (sb + selb) / ((scores_ms + select_ms) * 1e-3) / 1e9 / float(pk["hbm_gbs"])},
            "roofline": {"kernel": ("attn_tc_kernel (sfa_block_sparse_attn_rope)" if args.rope_on_load
                                    else "attn_tc_kernel (sfa_block_sparse_attn)"), "bound": "tensor",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{pk_src} bf16 burst",
                         "frac_of_sustained": achieved / float(pk.get("bf16_tflops_sustained", peak)),
                         "traffic": (tr["bytes_per_launch"] * (w.batch * w.heads_q * w.nb) / tr["tiles_per_launch"]
                                     if tr else None),
                         "traffic_note": (f"ncu DRAM bytes of one launch at {tr['workload']}, scaled by query tiles"
                                          if tr else "no capture for the current kernel source"),
                         "flops_per_launch": flops_step},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "upload and download streams, double-buffered device inputs and outputs",
                    "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                    "links_alone": {"h2d_GBps": h2d / (link_ms[0] * 1e-3) / 1e9,
                                    "ms_per_step_copies_both_ways": link_ms[1]}},
            "gpu_launches": (KERNELS_PER_STEP - (1 if args.fused else 0)) * K_,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            v, secs, text = oracle_head_sample(w, Q, K, V, h=0)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s",
                                    "cores": blas_threads() or len(os.sched_getaffinity(0)),
                                    "kind": "oracle", "sample": text, "seconds": secs, "cpu_model": cpu_model()}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
