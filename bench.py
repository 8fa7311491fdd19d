"""Benchmark of the hybrid sparse-attention layer prefill (one decoder layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long_128k]
    python bench.py --impl reference ...      # the fp64 CPU oracle, bounded sample

One step = one vnsa_forward over the whole layer (partition, pooling +
projection, compression attention + importance, top-k, selection, window + gate,
text GQA) on inputs already resident in HBM.  The inputs are larger than L2
(Q 0.94 GB, K and V 0.13 GB each at 128K), so no flush is needed between steps.
With N > 1 (torchrun) every rank runs its own independent prefill (its own
seeded sequence): weak scaling, no data-path collective; the time is the max
over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_long_block_b200.inputs import (WORKLOADS, cmp_mlp_weights,  # noqa: E402
                                                     gate_mlp_inputs, generate)

METRIC = "layer_prefill_tokens_per_s"
UNIT = "tokens/s"


def replica_workload(name, rank):
    """Weak scaling by independent replicas: rank r runs the named workload on
    its own synthetic sequence (seed + r); there is no data-path exchange."""
    base = WORKLOADS[name]
    return base.with_(seed=base.seed + rank)


def max_over_ranks(value, device):
    """Device-timed milliseconds, reduced to the slowest rank (the job time)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def algorithmic_work(wl, is_vision):
    """Algorithmic FLOPs per branch (4 d H_q per attended (query, key) pair)
    and the bytes of the HBM-bound steps (pooling; top-k: the fp32 importance
    of every visible block read once, the selection written), from the mask and
    config."""
    vis = np.nonzero(is_vision)[0]
    txt = np.nonzero(is_vision == 0)[0]
    nv = len(vis)
    B = wl.block
    st = wl.stride or B  # compression stride (overlapping blocks when below B)
    i = np.arange(nv, dtype=np.int64)
    nb = nv // B
    c = np.minimum((i + 1) // B, nb)  # complete selection blocks
    nc = (nv - B) // st + 1 if nv >= B else 0
    cc = np.where(i >= B - 1, np.minimum(nc, (i - B + 1) // st + 1), 0)  # visible cmp blocks
    own = i // B
    n_sel = np.minimum(wl.top_k, c + (own >= c).astype(np.int64))
    slc_tokens = B * (n_sel - 1) + (i % B + 1)
    swa_tokens = np.minimum(wl.window, i + 1)
    f = 4.0 * wl.d * wl.h_q
    es = 2 if wl.dtype == "bf16" else 4
    return {
        "cmp": f * float(cc.sum()),
        "slc": f * float(slc_tokens.sum()),
        "swa": f * float(swa_tokens.sum()),
        "text": f * float((txt.astype(np.int64) + 1).sum()),
        "pool_bytes": float(2 * (min(nv, (nc - 1) * st + B) if nc else 0) * wl.h_kv * wl.d * es
                            + 2 * nc * wl.h_kv * wl.d * es),
        "topk_bytes": float(4 * wl.h_kv * int(c.sum()) + 4 * wl.h_kv * nv * wl.top_k),
    }


def executed_work(wl, is_vision, idx):
    """Tensor FLOPs the attention kernels execute (every MMA of every tile,
    masked rows and keys included): 128-row tiles against 64-key tiles, 2 *
    128 * 64 * d flops per QK^T or P V product.  Compression: 16 queries per
    tile (8 head slots), a statistics pass (QK^T) and an exact pass (QK^T + P V)
    over the visible blocks; selection: 18 queries (7 heads) against the union
    of the 64-key tiles their selected blocks reach (from idx [h_kv][N_v][k]);
    with block 64 the tiles that only one, two or three of the 18 queries
    reach run tile-major instead, up to 18 such (query, tile) pairs per
    128-row tile; window and text: 18 queries against their key ranges.  (Up
    to 16 pairs per query leave the union: its single-query tiles, then the
    two-query and the three-query tiles while each of their queries has room,
    each in tile order.)"""
    prod = 2.0 * 128 * 64 * wl.d
    vis = np.nonzero(is_vision)[0]
    txt = np.nonzero(is_vision == 0)[0]
    nv, nb = len(vis), len(vis) // wl.block
    r = wl.h_q // wl.h_kv
    rpad = 1
    while rpad < r:
        rpad *= 2
    qc, qt = 128 // rpad, 128 // r
    cmp = slc = swa = text = 0.0
    B, st = wl.block, wl.stride or wl.block
    nc = (nv - B) // st + 1 if nv >= B else 0
    for q0 in range(0, nv, qc):
        ql = min(nv, q0 + qc) - 1
        vis_c = min(nc, (ql - B + 1) // st + 1) if ql >= B - 1 else 0
        t = -(-vis_c // 64)
        cmp += 3 * t
    single = np.zeros((wl.h_kv, (nv + 63) // 64 + 1), np.int64)  # pairs per (group, tile)
    for q0 in range(0, nv, qt):
        ql = min(nv, q0 + qt) - 1
        lo = max(0, q0 - wl.window + 1)
        swa += 2 * ((ql - lo + 64) // 64)
        for g in range(wl.h_kv):
            sel = idx[g, q0:ql + 1]
            if wl.block == 64:
                # up to 16 pairs per query leave the union: its single-query
                # tiles in tile order, then the two-query and then the
                # three-query tiles in tile order while each of the tile's
                # queries has a slot left
                who = {}
                for qi, row in enumerate(sel):
                    for j in row:
                        if j >= 0:
                            who.setdefault(int(j), []).append(qi)
                used = [0] * len(sel)
                pairs, leave = [], 0
                for j in sorted(who):
                    if len(who[j]) == 1 and used[who[j][0]] < 16:
                        used[who[j][0]] += 1
                        pairs.append(j)
                        leave += 1
                for share in (2, 3):
                    for j in sorted(who):
                        qs = who[j]
                        if len(qs) == share and all(used[q] < 16 for q in qs):
                            for q in qs:
                                used[q] += 1
                            pairs += [j] * share
                            leave += 1
                keep = len(who) - leave
                if pairs and keep:
                    slc += 2 * keep
                    np.add.at(single[g], pairs, 1)
                else:
                    slc += 2 * len(who)
                continue
            # the 64-key tiles each selected block reaches, up to the query
            ok = sel >= 0
            a = sel.astype(np.int64) * wl.block
            t0 = a // 64
            t1 = np.minimum(a + wl.block - 1, np.arange(q0, ql + 1)[:, None]) // 64
            span = int((t1 - t0)[ok].max()) if ok.any() else -1
            parts = [(t0 + o)[ok & (t0 + o <= t1)] for o in range(span + 1)]
            slc += 2 * (len(np.unique(np.concatenate(parts))) if parts else 0)
    slc += 2 * float((-(-single // qt)).sum())
    for x0 in range(0, len(txt), qt):
        xl = min(len(txt), x0 + qt) - 1
        text += 2 * ((int(txt[xl]) + 64) // 64)
    return {"cmp": wl.h_kv * cmp * prod, "slc": slc * prod, "swa": wl.h_kv * swa * prod,
            "text": wl.h_kv * text * prod}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = str(index)
        self.proc = None
        self.path = os.path.join("/tmp", f"vnsa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
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
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for _, _, fl in rows for k, v in enumerate(fl)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def smi_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return local_rank


def oracle_rates(wl, x, target_s=12.0, seed=1):
    """The fp64 oracle as it stands, timed on the host cores on bounded samples
    of the workload's rows.  Each oracle call pays a fixed cost (an fp64 copy
    of K/V and the pooling of every block) plus a cost per query row, which is
    far larger for a text row (dense over every earlier token) than for a
    vision row (its compressed blocks, selected blocks and window).  So the
    three are measured apart: one call of a single vision row gives the fixed
    cost, then a vision-row sample and a text-row sample (sized to share about
    target_s) give the per-row times.  The whole-layer estimate is
    T = fixed + N_v t_v + N_t t_t, and the rate reported is N / T."""
    import oracle
    p = oracle.OracleParams(h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                            top_k=wl.top_k, window=wl.window,
                            round_cmp_bf16=(wl.dtype == "bf16"))
    vis = np.nonzero(x["is_vision"])[0]
    txt = np.nonzero(x["is_vision"] == 0)[0]
    rng = np.random.default_rng(seed)

    def timed(rows):
        rows = np.sort(np.asarray(rows)).astype(np.int32)
        t0 = time.perf_counter()
        oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"], x["w_k"],
                       x["w_v"], rows=rows)
        return time.perf_counter() - t0

    fixed = min(timed(vis[-1:]), timed(vis[-1:]))
    share = 0.5 if len(txt) else 1.0

    def per_row(pool, probe):
        if len(pool) == 0:
            return 0.0, 0, 0.0
        n1 = min(len(pool), probe)
        t1 = max(timed(rng.choice(pool, n1, replace=False)) - fixed, 1e-6) / n1
        n2 = int(min(len(pool), max(n1, target_s * share / t1)))
        dt = timed(rng.choice(pool, n2, replace=False))
        return max(dt - fixed, 1e-9) / n2, n2, dt

    t_v, n_v, dt_v = per_row(vis, 64)
    t_t, n_t, dt_t = per_row(txt, 4)
    total = fixed + len(vis) * t_v + len(txt) * t_t
    return {"value": wl.n / total, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "fixed_s": fixed, "vision_row_ms": 1e3 * t_v, "text_row_ms": 1e3 * t_t,
            "layer_s_estimate": total,
            "sample": (f"fixed cost from one 1-row call ({fixed:.2f} s); {n_v} of {len(vis)} "
                       f"vision rows in {dt_v:.1f} s, {n_t} of {len(txt)} text rows in "
                       f"{dt_t:.1f} s (same inputs); value = N / (fixed + N_v t_v + N_t t_t)")}


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle, rank 0 only.  Each step is one
    bounded oracle measurement of the workload (fixed cost, a vision-row and a
    text-row sample, see oracle_rates); the line reports the mean whole-layer
    estimate of the timed steps."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    x = generate(wl)
    budget = max(1.0, float(args.ref_step_s))
    for w in range(args.warmup):
        oracle_rates(wl, x, target_s=budget, seed=100 + w)
    t0 = time.perf_counter()
    res = [oracle_rates(wl, x, target_s=budget, seed=200 + s_) for s_ in range(args.steps)]
    dt = time.perf_counter() - t0
    val = float(np.mean([r["value"] for r in res]))
    cpu = dict(res[-1])
    cpu["value"] = val
    cpu["steps_measured"] = len(res)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens": wl.n, "n_vision": wl.n_vision,
                       "n_text": wl.n_text, "top_k": wl.top_k, "window": wl.window},
            "cpu_baseline": cpu,
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# The other workloads of the method's evaluation settings, measured in the same
# process after the headline timing (outside its timed region): the
# Qwen2.5-VL-7B layer at 8K, the 36K training length and the global/local
# budget sweep at 64K (three top-k / window splits of about the same attended
# tokens per query).
PER_CONFIG = ("qwen_8k", "train_36k", "sweep_64k_k8_w1024", "sweep_64k_k16_w512",
              "sweep_64k_k32_w128")


def measure_config(wl, x, dev, steps=5, warmup=3):
    """ms per layer (device events over `steps` steps after `warmup`), stage
    times, and each branch's algorithmic FLOPs over its own time as a fraction
    of the measured bf16 peak."""
    import torch
    from sparse_attention_long_block_b200 import binding
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    q = torch.from_numpy(x["q"]).to(dev, td)
    k = torch.from_numpy(x["k"]).to(dev, td)
    v = torch.from_numpy(x["v"]).to(dev, td)
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    out = torch.empty_like(q)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        layer.forward(q, k, v, isv, gate, out=out, stream=stream)
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise SystemExit(f"device status error in {wl.name}")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        layer.forward(q, k, v, isv, gate, out=out, stream=stream)
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / steps
    layer.set_timing(True)
    stage = {}
    for _ in range(3):
        layer.forward(q, k, v, isv, gate, out=out, stream=stream)
        for kname, val in layer.timing().items():
            stage[kname] = stage.get(kname, 0.0) + val / 3
    layer.set_timing(False)
    torch.cuda.synchronize()
    path = layer.path()
    layer.close()
    del q, k, v, isv, gate, out
    torch.cuda.empty_cache()
    work = algorithmic_work(wl, x["is_vision"])
    pk = load_peaks()["bf16_tflops"]
    flops = work["cmp"] + work["slc"] + work["swa"] + work["text"]
    frac = {br: (work[br] / (stage[br] * 1e-3) / 1e12 / pk if stage.get(br) else None)
            for br in ("cmp", "slc", "swa", "text")}
    return {"tokens": wl.n, "top_k": wl.top_k, "window": wl.window, "kernels": path,
            "ms_per_layer": ms, "tokens_per_s": wl.n / (ms * 1e-3),
            "tensor_peak_frac": flops / (ms * 1e-3) / 1e12 / pk,
            "branch_ms": {kk: stage.get(kk, 0.0) for kk in
                          ("partition", "pool", "cmp", "topk", "slc", "swa", "text")},
            "branch_tensor_frac": frac,
            "algorithmic_gflop": {br: work[br] / 1e9 for br in ("cmp", "slc", "swa", "text")},
            "steps": steps, "warmup": warmup}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="long_128k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="vnsa", choices=["vnsa", "reference"])
    ap.add_argument("--mode", default="prefill", choices=["prefill", "decode"],
                    help="decode: time single-token steps after a prefill of the rest")
    ap.add_argument("--decode-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ref-step-s", type=float, default=6.0,
                    help="oracle seconds per reference-arm step (bounded sample)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads' measurements after the headline")
    ap.add_argument("--traffic-json", default=os.path.join(ROOT, "profiles", "traffic.json"))
    ap.add_argument("--mlp", action="store_true",
                    help="each step also computes the gate logits from the layer input "
                         "through the gate perceptron, and compression uses its perceptron")
    ap.add_argument("--gate-hidden", type=int, default=256)
    ap.add_argument("--cmp-hidden", type=int, default=128)
    ap.add_argument("--cmp-stride", type=int, default=0,
                    help="compression stride below the block size (overlapping blocks); 0: the block")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.mode == "decode":
        run_decode_bench(args, rank, world, local_rank)
        return

    import torch
    import torch.distributed as dist
    from sparse_attention_long_block_b200 import binding

    if not torch.cuda.is_available():
        raise SystemExit("bench needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dist_on = world > 1
    if dist_on:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    wl = replica_workload(args.workload, rank)
    if args.cmp_stride:
        wl = wl.with_(stride=args.cmp_stride)
    x = generate(wl)
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dev = torch.device("cuda", local_rank)
    q = torch.from_numpy(x["q"]).to(dev, td)
    k = torch.from_numpy(x["k"]).to(dev, td)
    v = torch.from_numpy(x["v"]).to(dev, td)
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    out = torch.empty_like(q)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype, stride=wl.stride)
    stream = torch.cuda.current_stream()
    gm = None
    if args.mlp:
        # the perceptrons: gate logits from the layer input x [n][h_q d] each
        # step (into the gate buffer the layer reads), compression through its
        # perceptron
        gi = gate_mlp_inputs(wl, wl.h_q * wl.d, args.gate_hidden, seed=200 + rank)
        gm = {kk: torch.from_numpy(vv).to(dev, td if kk in ("x", "g1", "g2") else torch.float32)
              for kk, vv in gi.items()}
        del gi
        layer.set_cmp_mlp({kk: torch.from_numpy(vv)
                           for kk, vv in cmp_mlp_weights(wl, args.cmp_hidden).items()})

    def gate_step():
        layer.gate_mlp(gm["x"], gm["g1"], gm["c1"], gm["g2"], gm["c2"], out=gate, stream=stream)

    def step():
        if gm is not None:
            gate_step()
        layer.forward(q, k, v, isv, gate, out=out, stream=stream)

    def barrier():
        if dist_on:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise SystemExit("device status error during warm-up")
    launches_per_step = layer.launches()
    if gm is not None:
        gate_step()
        torch.cuda.synchronize()
        launches_per_step += layer.launches()

    sampler = ClockSampler(smi_index(local_rank)) if rank == 0 else None
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    ev1.synchronize()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    ms = ev0.elapsed_time(ev1) / max(args.steps, 1)
    if dist_on:
        ms = max_over_ranks(ms, dev)
    if layer.device_status() != 0:
        raise SystemExit("device status error in the timed region")

    # per-stage times (library events on the same stream), outside the timed region
    layer.set_timing(True)
    stage_ms = {}
    reps = 3
    for _ in range(reps):
        step()
        for kname, val in layer.timing().items():
            stage_ms[kname] = stage_ms.get(kname, 0.0) + val / reps
    layer.set_timing(False)
    torch.cuda.synchronize()
    executed = None
    if wl.dtype == "bf16" and wl.d == 128:
        dbg, tens = binding.make_debug(wl.n, wl.h_q, wl.h_kv, wl.d, wl.top_k, wl.block,
                                       dtype=td, want=("idx",), stride=wl.stride)
        layer.forward(q, k, v, isv, gate, out=out, dbg=dbg, stream=stream)
        torch.cuda.synchronize()
        nvis = int(x["is_vision"].sum())
        executed = executed_work(wl, x["is_vision"], tens["idx"][:, :nvis].cpu().numpy())
        del tens

    # the gate perceptron alone (same stream, after warm-up), for its roofline
    gate_mlp = None
    if gm is not None:
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ga.record(stream)
        for _ in range(args.steps):
            gate_step()
        gb.record(stream)
        gb.synchronize()
        g_ms = ga.elapsed_time(gb) / max(args.steps, 1)
        dm, hid, n_out = wl.h_q * wl.d, args.gate_hidden, 3 * wl.h_q
        es = 2 if wl.dtype == "bf16" else 4
        g_bytes = wl.n * dm * es + (dm * hid + hid * n_out) * es + wl.n * n_out * 4
        g_flops = 2.0 * wl.n * (dm * hid + hid * n_out)
        pk = load_peaks()
        gate_mlp = {"ms": g_ms, "d_model": dm, "hidden": hid, "bytes": g_bytes,
                    "flops": g_flops,
                    "hbm_gbs": g_bytes / (g_ms * 1e-3) / 1e9,
                    "hbm_frac": g_bytes / (g_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                    "tflops": g_flops / (g_ms * 1e-3) / 1e12,
                    "tensor_frac": g_flops / (g_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                    "bound": ("hbm" if g_bytes / pk["hbm_gbs"] / 1e9 >
                              g_flops / pk["bf16_tflops"] / 1e12 else "tensor")}

    # end to end through the C ABI with host buffers (pinned)
    e2e = None
    if not args.no_e2e and gm is None:
        hq = torch.from_numpy(x["q"]).to(td).pin_memory()
        hk = torch.from_numpy(x["k"]).to(td).pin_memory()
        hv = torch.from_numpy(x["v"]).to(td).pin_memory()
        hi = torch.from_numpy(x["is_vision"]).pin_memory()
        hg = torch.from_numpy(x["gate"]).pin_memory()
        ho = torch.empty_like(hq).pin_memory()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # (1) one synchronous call per step (vnsa_forward_host): copies in,
        # layer, copy out, host waits; no overlap between steps
        layer.forward_host(hq, hk, hv, hi, hg, ho, stream=stream)
        s_steps = max(2, min(args.steps, 5))
        barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(s_steps):
            layer.forward_host(hq, hk, hv, hi, hg, ho, stream=stream)
        b.record(stream)
        b.synchronize()
        sync_ms = a.elapsed_time(b) / s_steps
        # (2) streamed calls (vnsa_forward_host_async): every step still copies
        # its inputs in and its output out, and the copies of neighbouring
        # steps overlap the layer in between; the timed region runs from
        # before the first input copy to after the last output copy
        layer.wait_host(layer.forward_host_async(hq, hk, hv, hi, hg, ho, stream=stream))
        e_steps = max(3, args.steps)
        barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(e_steps):
            tk = layer.forward_host_async(hq, hk, hv, hi, hg, ho, stream=stream)
        layer.join_host(stream)
        b.record(stream)
        b.synchronize()
        layer.wait_host(tk)
        e_ms = a.elapsed_time(b) / e_steps
        if dist_on:
            e_ms = max_over_ranks(e_ms, dev)
            sync_ms = max_over_ranks(sync_ms, dev)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hi, hg))
        e2e = {"value": world * wl.n / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": ho.numel() * ho.element_size(), "ms_per_step": e_ms,
               "steps": e_steps,
               "api": "vnsa_forward_host_async: pinned host buffers, two device staging "
                      "slots, copies of neighbouring steps overlap the layer",
               "sync_call": {"api": "vnsa_forward_host", "ms_per_step": sync_ms,
                             "value": world * wl.n / (sync_ms / 1e3)}}

    work = algorithmic_work(wl, x["is_vision"])
    flops = work["cmp"] + work["slc"] + work["swa"] + work["text"]
    peaks = load_peaks()
    branch_ms = {"partition": stage_ms.get("partition", 0.0), "pool": stage_ms.get("pool", 0.0),
                 "cmp": stage_ms.get("cmp", 0.0), "topk": stage_ms.get("topk", 0.0),
                 "slc": stage_ms.get("slc", 0.0), "swa": stage_ms.get("swa", 0.0),
                 "text": stage_ms.get("text", 0.0)}
    flop_of = {"cmp": work["cmp"], "slc": work["slc"], "swa": work["swa"], "text": work["text"]}
    # the vision kernel of the SIMT path does selection + window in one stage
    if branch_ms["slc"] == 0.0 and branch_ms["swa"] > 0.0:
        flop_of["swa"] = work["slc"] + work["swa"]
        flop_of["slc"] = 0.0
    dom = max(flop_of, key=lambda s: branch_ms.get(s, 0.0))
    dom_ms = branch_ms[dom]
    achieved = flop_of[dom] / (dom_ms * 1e-3) / 1e12 if dom_ms > 0 else 0.0
    traffic = None
    try:
        with open(args.traffic_json) as f:
            tj = json.load(f)
        ent = tj.get(wl.name, {}).get(dom)
        if ent and ent.get("kernel_build") == layer_build_id():
            traffic = ent["bytes_per_launch"]
    except Exception:
        pass
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                "peak_source": peaks["source"] + " burst bf16"}
    pool_gbs = work["pool_bytes"] / (branch_ms["pool"] * 1e-3) / 1e9 if branch_ms["pool"] else 0
    topk_gbs = work["topk_bytes"] / (branch_ms["topk"] * 1e-3) / 1e9 if branch_ms["topk"] else 0
    value = world * wl.n / (ms / 1e3)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_rates(wl, x)
    if dist_on:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "tokens": wl.n, "n_vision": wl.n_vision,
                       "n_text": wl.n_text, "h_q": wl.h_q, "h_kv": wl.h_kv, "d": wl.d,
                       "block": wl.block, "cmp_stride": wl.stride or wl.block,
                       "top_k": wl.top_k, "window": wl.window,
                       "attention": "dense (all tokens text)" if wl.dense else "hybrid",
                       "kernels": layer.path(),
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (no flush)",
                       "perceptrons": None if gm is None else {
                           "gate": f"x [{wl.n}][{wl.h_q * wl.d}] -> {args.gate_hidden} -> "
                                   f"{3 * wl.h_q} logits, every step",
                           "compression_hidden": args.cmp_hidden}},
            "tensor_peak_frac": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "executed": None if executed is None else {
                "tflop": {kk: vv / 1e12 for kk, vv in executed.items()},
                "tflops_per_s": sum(executed.values()) / (ms * 1e-3) / 1e12,
                "frac_of_peak": sum(executed.values()) / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                "slc_frac_of_peak": (executed["slc"] / (branch_ms["slc"] * 1e-3) / 1e12 /
                                     peaks["bf16_tflops"]) if branch_ms["slc"] else None},
            "algorithmic_gflop": {kk: vv / 1e9 for kk, vv in flop_of.items()},
            "branch_ms": branch_ms,
            "pool_hbm": {"achieved_gbs": pool_gbs, "peak_gbs": peaks["hbm_gbs"],
                         "frac": pool_gbs / peaks["hbm_gbs"]},
            "topk_hbm": {"achieved_gbs": topk_gbs, "peak_gbs": peaks["hbm_gbs"],
                         "frac": topk_gbs / peaks["hbm_gbs"], "bytes": work["topk_bytes"],
                         "stage": "top-k and the selection-union launches"},
            "roofline": roofline,
            "gate_mlp": gate_mlp,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
    layer.close()
    if rank == 0:
        if world == 1 and not args.no_per_config and args.workload == "long_128k":
            del q, k, v, isv, gate, out
            torch.cuda.empty_cache()
            per = {}
            xs = None
            for name in PER_CONFIG:
                cw = WORKLOADS[name]
                if name.startswith("sweep_64k"):
                    # the three budget splits share one input sequence
                    xs = xs if xs is not None else generate(cw)
                    xc = xs
                else:
                    xc = generate(cw)
                per[name] = measure_config(cw, xc, dev)
            line["per_config"] = per
        print(json.dumps(line), flush=True)
    if dist_on:
        dist.destroy_process_group()


def decode_bytes(wl, i, kind):
    """Algorithmic HBM bytes of one decode step: block keys/values of the
    visible blocks, the selected blocks' and the window's K/V rows (vision), or
    every K/V row (text), plus q, gates and the output row."""
    es = 2 if wl.dtype == "bf16" else 4
    row = wl.h_kv * wl.d * es
    io = 2 * wl.h_q * wl.d * es + wl.h_q * 3 * 4
    if kind == "text":
        return 2 * (i + 1) * row + io
    c = (i + 1) // wl.block
    sel = min(wl.top_k, c + 1) * wl.block
    return 2 * c * row + 2 * sel * row + 2 * min(wl.window, i + 1) * row + io


def run_decode_bench(args, rank, world, local_rank):
    """Decode steps of the named workload's stream: the last D tokens are moved
    to the end of the vision run (so they decode through the sparse branches),
    the rest is prefilled once, then D single-token steps are timed on the
    device; the first `warmup` steps of a second pass are untimed."""
    import torch
    from sparse_attention_long_block_b200 import binding
    base = replica_workload(args.workload, rank)
    D = args.decode_tokens
    nv, nt = base.n_vision, base.n_text
    mask = np.concatenate([np.ones(nv - D, np.uint8), np.zeros(nt, np.uint8),
                           np.ones(D, np.uint8)])
    wl = base.with_(name=base.name)
    x = generate(wl, is_vision=mask)
    torch.cuda.set_device(local_rank)
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dev = torch.device("cuda", local_rank)
    q = torch.from_numpy(x["q"]).to(dev, td)
    k = torch.from_numpy(x["k"]).to(dev, td)
    v = torch.from_numpy(x["v"]).to(dev, td)
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    n = wl.n
    n0 = n - D
    layer = binding.Layer(n_max=n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype)
    qs = [q[t].contiguous() for t in range(n0, n)]
    gs = [gate[t].contiguous() for t in range(n0, n)]
    outs = [torch.empty_like(qs[0]) for _ in range(D)]
    stream = torch.cuda.current_stream()

    def prefill():
        layer.forward(q[:n0].contiguous(), k[:n0].contiguous(), v[:n0].contiguous(),
                      isv[:n0].contiguous(), gate[:n0].contiguous(), stream=stream)

    def steps(lo, hi):
        for j in range(lo, hi):
            layer.decode(n0 + j + 1, qs[j], k, v, isv, gs[j], out=outs[j], stream=stream)

    prefill()
    steps(0, D)  # warm-up pass
    prefill()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    steps(0, D)
    ev1.record(stream)
    ev1.synchronize()
    if layer.device_status() != 0:
        raise SystemExit("device status error in the decode steps")
    ms = ev0.elapsed_time(ev1) / D
    launches = layer.launches()
    peaks = load_peaks()
    i0 = nv - D
    nbytes = float(np.mean([decode_bytes(wl, i0 + j, "vision") for j in range(D)]))
    gbs = nbytes / (ms * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": "decode_tokens_per_s", "value": world * 1e3 / ms, "unit": "tokens/s",
            "n_gpus": world, "steps": D, "warmup": D, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "mode": "decode (vision tokens)", "context": n,
                       "decoded": D, "top_k": wl.top_k, "window": wl.window},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "bytes_per_step": nbytes},
            "gpu_launches": launches * D,
        }
        print(json.dumps(line), flush=True)
    layer.close()


# the sources that define the tensor-core attention kernel and its launches
ATTN_KERNEL_SOURCES = ("tc_attn.cu", "tc_attn.h", "sgl_attn.cu", "sgl_attn.h", "tc_ptx.cuh",
                       "common.cuh", "kernels.h", "config.h")


def layer_build_id():
    """Identity of the attention kernel's sources (a hash of the files that
    define it) for stored traffic records: a record taken on another build of
    that kernel is not reported."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_long_block_b200", "csrc")
    for name in ATTN_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
