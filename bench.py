#!/usr/bin/env python
"""Benchmark of the orthonormalized-update optimizer step on B200.

Workload (one "step"): a Llama-3-8B-shaped parameter set -- 32 layers x
{q, o 4096x4096; k, v 1024x4096; gate, up 14336x4096; down 4096x14336}, 224
matrices, 6,979,321,856 parameters -- with bf16 gradients N(0, 0.01^2) plus a
rank-32 spike, fp32 momentum and bf16 weights.  One step is the whole hot
path through the library's C ABI:

  dion_momentum_update (error-feedback buffer B = M + G, float64 row keys)
  dion3_select_rows    (top 1/8 rows by row norm, gather + scale, M[S] = mu B[S])
  gram_ns_orthogonalize(5 iterations, restart after 3, bf16 / tf32 tensor cores)
  apply_update         (W[S] -= lr * scale * O)

Prints one JSON line (rank 0).  ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "optimizer-step ms (8B-shaped param set) & Gram-NS TFLOP/s vs BF16 peak, 1×B200"
RHO = 0.125
MU = 0.95
LR = 0.02
ITERS = 5
RESTART_AFTER = (3,)
CHUNK_LAYERS = 4  # end-to-end schedule: layers per host-to-device chunk
# tf32 / bf16 dense tensor throughput ratio (nominal 1.1 / 2.25 PFLOP/s)
TF32_RATIO = 1.1 / 2.25
# tensor-core GEMM kinds reported by the library's launch timing
KIND_NAMES = {0: "bf16 K-major", 1: "bf16 MN-major (Q X)", 2: "tf32 K-major",
              3: "tf32 MN-major", 4: "bf16 symmetric (X X^T)", 5: "bf16 symmetric MN",
              6: "tf32 symmetric (k x k products)", 7: "tf32 symmetric MN"}


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dion", action="store_true",
                    help="skip the Dion / Orth-Dion measurements of the JSON line")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the standard-vs-Gram crossover points of the JSON line")
    ap.add_argument("--cpu-sample-layers", type=int, default=1)
    ap.add_argument("--micro", choices=["gram", "dion", "dion_set"], default=None,
                    help="one kernel-level case for profiling: Gram NS on --nb blocks "
                         "of --m x --n bf16, one Dion / Orth-Dion matrix --m x --n "
                         "at --rank (--mode colnorm|qr), or the 8B-shaped set of "
                         "--layers layers in one grouped Dion / Orth-Dion call")
    ap.add_argument("--nb", type=int, default=32)
    ap.add_argument("--m", type=int, default=1792)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--rank", type=int, default=256)
    ap.add_argument("--mode", choices=["colnorm", "qr"], default="qr")
    ap.add_argument("--sweep", action="store_true",
                    help="shape sweep instead of the step: standard vs Gram NS over "
                         "m in 512..8192, n/m in 1, 4, 16; Dion / Orth-Dion over rank "
                         "64..1024 on 4096x4096 (one JSON line)")
    return ap.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _traffic():
    """DRAM bytes per launch from the committed ncu launch-list summary,
    keyed by kernel; an entry counts only while the kernel's source hash
    still matches the one the counters were taken with."""
    import hashlib
    csrc = os.path.join(ROOT, "orthonormalized_update_optimizers_b200", "csrc")

    def digest(*names):
        h = hashlib.sha256()
        for nm in names:
            with open(os.path.join(csrc, nm), "rb") as f:
                h.update(f.read())
        return h.hexdigest()[:16]

    current = {"umma_gemm_kernel tf32 symmetric": digest("gemm_umma.cu", "umma.cuh"),
               "momentum_kernel": digest("momentum.cu")}
    out = {}
    try:
        with open(os.path.join(ROOT, "profiles", "launches_llama8b_dion3_gram_ns_step.md")) as f:
            for line in f:
                parts = [p.strip() for p in line.strip().strip("|").split("|")]
                if len(parts) == 3 and parts[0] in current and parts[1].isdigit():
                    if parts[2] == current[parts[0]]:
                        out[parts[0]] = int(parts[1])
    except OSError:
        pass
    return out


def gram_ns_flops(k: int, n: int, iters: int = ITERS, restarts=RESTART_AFTER):
    """Algorithmic flops of Gram NS on a k x n block (k <= n after
    orientation), split into bf16 (k x n products) and tf32 (k x k symmetric
    products).  Symmetric outputs count the upper triangle only."""
    if k > n:
        k, n = n, k
    syrk = k * (k + 1) * n           # X X^T, triangle
    qx = 2 * k * k * n               # Q X
    sym = k * k * (k + 1)            # symmetric k x k product, triangle
    bf, tf = syrk, 0
    q_identity = True
    for t in range(1, iters + 1):
        tf += sym                    # A^2 inside H
        if not q_identity:
            tf += sym                # H Q
        q_identity = False
        if t == iters:
            break
        if t in restarts:
            bf += qx + syrk
            q_identity = True
        else:
            tf += 2 * sym            # H (H A)
    bf += qx
    return bf, tf


def std_ns_flops(k: int, n: int, iters: int = ITERS):
    """Algorithmic flops of the standard quintic iteration on a k x n block
    (k <= n after orientation): per iteration the triangle of X X^T, the
    triangle of the symmetric b A + c A^2, and the dense a X + B X."""
    if k > n:
        k, n = n, k
    return iters * (k * (k + 1) * n + k * k * (k + 1) + 2 * k * k * n)


def _workload_shapes(layers):
    from orthonormalized_update_optimizers_b200 import synth
    return synth.llama8b_shapes(layers)


# ----------------------------------------------------------------- reference

def run_reference(args):
    """Time the float64 oracle, as it stands, on a bounded sample: W warm-up
    repetitions on one small matrix, then K timed repetitions of the layer
    sample, each scaled to the full parameter set."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    t_warm = time.perf_counter()
    for _ in range(args.warmup):
        _oracle_sample(args, n_matrices=1, first=1)  # k projection, 1024 x 4096
    t_warm = time.perf_counter() - t_warm
    per_step, measured = [], []
    for _ in range(args.steps):
        per_step.append(cpu_baseline(args)["value"])
        measured.append(cpu_baseline.last_seconds)
    ms = statistics.median(per_step)
    line = cpu_baseline.last
    line = dict(line, value=round(ms, 3))
    out = {
        "impl": "reference", "metric": METRIC, "value": round(ms, 3),
        "unit": "ms", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": _config(args.layers, args.gpus),
        "cpu_baseline": line,
        "e2e": {"value": round(ms, 3), "unit": "ms", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        # what actually ran: each "step" is one sample of 7 * cpu_sample_layers
        # matrices, timed and scaled to the whole parameter set
        "samples_run": {"count": args.steps, "matrices_each": 7 * args.cpu_sample_layers,
                        "scale_each": len(_workload_shapes(args.layers)) /
                                      (7 * args.cpu_sample_layers),
                        "measured_s": [round(x, 3) for x in measured],
                        "measured_s_total": round(sum(measured), 3),
                        "warmup_s": round(t_warm, 3)},
    }
    print(json.dumps(out), flush=True)


def _oracle_sample(args, n_matrices, first=0):
    """Seconds the oracle's Dion3 step takes on matrices first..first+n-1 of
    the workload (inputs from the shared seeded generator, on the host)."""
    import numpy as np
    import torch
    from orthonormalized_update_optimizers_b200 import synth
    from oracle import dion3 as odion3

    shapes = _workload_shapes(args.layers)
    t_total = 0.0
    for i in range(first, first + n_matrices):
        _, m, n = shapes[i]
        G = synth.lowrank_plus_noise(m, n, 32, 0.01, synth.seed_for(3, i),
                                     torch.bfloat16, "cpu")
        G64 = G.float().numpy().astype(np.float64)
        M = np.zeros((m, n), dtype=np.float32)
        W = synth.gaussian((m, n), synth.seed_for(3, 1000 + i), 0.02,
                           torch.bfloat16, "cpu").float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        odion3.dion3_step(M, G64, W, MU, RHO, LR, 1.0, iters=ITERS,
                          restart_after=RESTART_AFTER)
        t_total += time.perf_counter() - t0
    return t_total


def cpu_baseline(args):
    """Oracle Dion3 step on the first `cpu_sample_layers` layers' matrices
    (same generator, same seeds), scaled to the full parameter set by the
    number of matrices.  Returns the cpu_baseline object."""
    shapes = _workload_shapes(args.layers)
    n_sample = 7 * args.cpu_sample_layers
    t_total = _oracle_sample(args, n_sample)
    scale = len(shapes) / n_sample
    ms = t_total * 1e3 * scale
    cores = len(os.sched_getaffinity(0))
    line = {"value": round(ms, 3), "unit": "ms", "cores": cores, "kind": "oracle",
            "sample": f"float64 NumPy oracle Dion3 step on the {n_sample} matrices of "
                      f"layer(s) 0..{args.cpu_sample_layers - 1}, measured {t_total:.2f} s, "
                      f"extrapolated x{scale:g} to all {len(shapes)} matrices",
            "extrapolated": scale != 1.0}
    cpu_baseline.last = line
    cpu_baseline.last_seconds = t_total
    return line


def _config(layers, world=1):
    shapes = _workload_shapes(layers)
    params = sum(m * n for _, m, n in shapes)
    return {"workload": f"Llama-3-8B-shaped optimizer step ({layers} layers, {len(shapes)} "
                        "matrices): Dion3 rho=1/8 with error feedback + Gram Newton-Schulz "
                        "(5 iterations, restart after 3), bf16 gradients N(0,0.01^2)+rank-32 "
                        "spike, fp32 momentum, bf16 weights",
            "params": params, "matrices": len(shapes), "rho": RHO, "mu": MU,
            "l2": "inputs larger than L2 (about 56 GB resident per step)",
            "parallelism": "single GPU" if world == 1 else
                           f"dp{world}: per-matrix partition of the step across {world} GPUs, "
                           "NCCL all-gather of the kept-row updates, every rank updates "
                           "all weights"}


# ----------------------------------------------------------------------- ours

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def run_ours(args):
    import numpy as np
    import torch
    import orthonormalized_update_optimizers_b200 as ouo
    from orthonormalized_update_optimizers_b200 import shard, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)

    shapes = _workload_shapes(args.layers)
    mn = [(m, n) for _, m, n in shapes]
    # Per-matrix partition: this rank steps its own matrices, the kept-row
    # updates are all-gathered, every rank updates all its weights.  With one
    # rank the plan is everything and the exchange is nothing.
    parts = shard.plan_partition(mn, world, RHO)
    own = parts[rank]
    lay = shard.ExchangeLayout(mn, parts, RHO)
    # every operand laid out one block per shape (the layout the grouped
    # launches read without copies)
    own_mn = [mn[i] for i in own]
    Gs = ouo.batch_empty(own_mn, torch.bfloat16, dev)
    Ms = ouo.batch_empty(own_mn, torch.float32, dev)
    for k, i in enumerate(own):
        m, n = mn[i]
        Gs[k].copy_(synth.lowrank_plus_noise(m, n, 32, 0.01, synth.seed_for(3, i),
                                             torch.bfloat16, dev))
        Ms[k].zero_()
    Ws = ouo.batch_empty(mn, torch.bfloat16, dev)
    for i, (m, n) in enumerate(mn):
        Ws[i].copy_(synth.gaussian((m, n), synth.seed_for(3, 1000 + i), 0.02,
                                   torch.bfloat16, dev))
    ks = [lay.k[i] for i in own]
    assert ks == [ouo.dion3_num_selected(mn[i][0], RHO) for i in own]
    keys = torch.empty(max(1, sum(mn[i][0] for i in own)), dtype=torch.float64, device=dev)
    payload = torch.empty(max(1, lay.payload_bytes), dtype=torch.uint8, device=dev)
    gathered = payload if world == 1 else torch.empty(world * lay.payload_bytes,
                                                      dtype=torch.uint8, device=dev)
    idx, O = lay.views(payload, rank)  # selection and Gram NS write the payload
    kn = [(k, mn[i][1]) for k, i in zip(ks, own)]
    X0 = ouo.batch_empty(kn, torch.bfloat16, dev)
    scale = torch.empty(max(1, len(own)), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    Mb, Gb = ouo.MatBatch(Ms), ouo.MatBatch(Gs)
    Xb, Ob = ouo.MatBatch(X0), ouo.MatBatch(O)
    params = ouo.ns_params(iters=ITERS, restart_after=RESTART_AFTER, normalize=False)
    ws = torch.empty(max(1, ouo.gram_ns_workspace_bytes(Xb, params) if own else 1),
                     dtype=torch.uint8, device=dev)
    # Muon-style per-matrix update scale sqrt(max(1, rows / cols))
    scales = [math.sqrt(max(1.0, m / n)) for m, n in mn]
    # one weight-update call per source rank, on its segment of the exchange
    segs = []
    for r, (gidx, gO) in enumerate(lay.gathered_views(gathered)):
        if parts[r]:
            segs.append((ouo.MatBatch([Ws[i] for i in parts[r]]), ouo.MatBatch(gO), gidx,
                         [scales[i] for i in parts[r]]))

    def step():
        if own:
            ouo.dion_momentum_update(Mb, Gb, MU, "accum", keys)
            ouo.dion3_select_rows(Mb, keys, RHO, idx, Xb, scale, ef=True, mu=MU)
            ouo.gram_ns_orthogonalize(Xb, Ob, params, workspace=ws, status=status)
        exchange_and_update()

    def exchange_and_update():
        shard.all_gather_payload(payload, gathered)
        for Wb_r, Ob_r, idx_r, sc_r in segs:
            ouo.apply_update(Wb_r, Ob_r, LR, idx=idx_r, scale=sc_r)

    # The same step in chunks of CHUNK_LAYERS layers, for the end-to-end
    # measurement: each chunk's gradients arrive from the host on a copy
    # stream while the previous chunk is being stepped.  Every per-chunk
    # operand is a view of the whole-step buffers (row keys, kept indices,
    # scales, X0 and O are laid out in matrix order), so a chunked step
    # computes exactly what step() does.
    chunk_size = 7 * CHUNK_LAYERS
    chunks = []
    kpos = np.concatenate([[0], np.cumsum(ks)]).astype(int) if own else [0]
    rpos = np.concatenate([[0], np.cumsum([mn[i][0] for i in own])]).astype(int) if own else [0]
    for c0 in range(0, len(own), chunk_size):
        c1 = min(len(own), c0 + chunk_size)
        sl = slice(c0, c1)
        chunks.append({
            "G": Gs[sl], "Mb": ouo.MatBatch(Ms[sl]), "Gb": ouo.MatBatch(Gs[sl]),
            "Xb": ouo.MatBatch(X0[sl]), "Ob": ouo.MatBatch(O[sl]),
            "keys": keys[rpos[c0]:rpos[c1]], "idx": idx[kpos[c0]:kpos[c1]],
            "scale": scale[c0:c1]})

    def step_chunk(ch):
        ouo.dion_momentum_update(ch["Mb"], ch["Gb"], MU, "accum", ch["keys"])
        ouo.dion3_select_rows(ch["Mb"], ch["keys"], RHO, ch["idx"], ch["Xb"], ch["scale"],
                              ef=True, mu=MU)
        # chunks run one after another on one stream and share the workspace
        # sized for the whole step
        ouo.gram_ns_orthogonalize(ch["Xb"], ch["Ob"], params, workspace=ws, status=status)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x):
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(args.warmup):
        step()
    barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    n0 = ouo.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    barrier()
    launches = ouo.launch_count() - n0
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    # --- the step's parts, timed inside full steps: events recorded between
    # the calls of each step, so the parts add up to the step
    part_names = ("momentum", "selection", "gram_ns", "update")
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for k in range(args.steps):
        ev = pev[k]
        ev[0].record()
        if own:
            ouo.dion_momentum_update(Mb, Gb, MU, "accum", keys)
        ev[1].record()
        if own:
            ouo.dion3_select_rows(Mb, keys, RHO, idx, Xb, scale, ef=True, mu=MU)
        ev[2].record()
        if own:
            ouo.gram_ns_orthogonalize(Xb, Ob, params, workspace=ws, status=status)
        ev[3].record()
        exchange_and_update()
        ev[4].record()
    barrier()
    part_ms = {}
    for j, nm in enumerate(part_names):
        part_ms[nm] = max_over_ranks(
            sum(pev[k][j].elapsed_time(pev[k][j + 1]) for k in range(args.steps)) / args.steps)
    mom_ms, sel_ms = part_ms["momentum"], part_ms["selection"]
    gram_ms, app_ms = part_ms["gram_ns"], part_ms["update"]
    # --- per-launch timing of every tensor-core GEMM launch of full steps
    # (CUDA events recorded by the library around each launch, on its stream)
    ouo.timing_enable(True)
    for _ in range(args.steps):
        step()
    barrier()
    kinds = {}
    for kind, name in KIND_NAMES.items():
        n, kms, fl = ouo.timing_read(kind)
        if n:
            kinds[name] = {"launches_per_step": n // args.steps,
                           "ms_per_step": round(kms / args.steps, 4),
                           "avg_launch_us": round(1e3 * kms / n, 2),
                           "tflops": round(fl / (kms * 1e-3) / 1e12, 1)}
    ouo.timing_enable(False)
    clocks = sampler.stop()
    st = int(status.item())

    peaks = _peaks()
    # Gram-NS flops of the whole job (all ranks' matrices) over the slowest
    # rank's Gram-NS time
    bf = tf = 0
    for i, (m, n) in enumerate(mn):
        b_, t_ = gram_ns_flops(lay.k[i], n)
        bf += b_
        tf += t_
    flops = bf + tf
    tflops = flops / (gram_ms * 1e-3) / 1e12
    # effective peak of the bf16 / tf32 mix (each at its own dtype's peak)
    p_bf = peaks["bf16_tflops"]
    p_tf = p_bf * TF32_RATIO
    peak_eff = flops / (bf / p_bf + tf / p_tf)
    all_kn = [(lay.k[i], mn[i][1]) for i in range(len(mn))]
    # momentum kernel of this rank (its own matrices)
    elems = sum(mn[i][0] * mn[i][1] for i in own)
    rows = sum(mn[i][0] for i in own)
    mom_bytes = elems * (4 + 2 + 4) + rows * 8   # read M, G; write M; write keys
    mom_gbs = mom_bytes / (mom_ms * 1e-3) / 1e9 if mom_ms > 0 else 0.0
    mom_launches = -(-len(own) // 128)
    # The dominant kernel of the step by device time: a GEMM kind or the
    # momentum kernel.  The step lasts tens of milliseconds, far shorter than
    # the seconds-long loop the sustained peak was taken in, so the burst
    # dense-bf16 peak is the denominator (tf32 at the nominal tf32/bf16
    # ratio); the sustained one is reported beside it.
    p_bf_s = peaks["bf16_tflops_sustained"]
    traffic = _traffic()
    dom_name, dom = max(kinds.items(), key=lambda kv: kv[1]["ms_per_step"]) if kinds else (None, None)
    if dom is not None and dom["ms_per_step"] > mom_ms:
        is_tf32 = "tf32" in dom_name
        ratio = TF32_RATIO if is_tf32 else 1.0
        peak = p_bf * ratio
        peak_s = p_bf_s * ratio
        roofline = {"bound": "tensor", "kernel": f"umma_gemm_kernel ({dom_name})",
                    "achieved": dom["tflops"], "peak": round(peak, 1), "unit": "TFLOP/s",
                    "frac": round(dom["tflops"] / peak, 4),
                    "traffic": traffic.get("umma_gemm_kernel tf32 symmetric")
                    if "tf32 symmetric" in dom_name else None,
                    "peak_note": f"{'tf32 = ' if is_tf32 else ''}burst bf16 {p_bf}"
                                 f"{' x 0.489 nominal tf32/bf16' if is_tf32 else ''} "
                                 f"({peaks['source']}); tf32 is not measured on its own",
                    "peak_sustained": round(peak_s, 1),
                    "frac_of_sustained": round(dom["tflops"] / peak_s, 4),
                    "units": "algorithmic flops per launch (symmetric outputs: upper "
                             "triangle) / CUDA-event launch time"}
    else:
        roofline = {"bound": "hbm", "kernel": "momentum_kernel", "achieved": round(mom_gbs, 1),
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(mom_gbs / peaks["hbm_gbs"], 4),
                    "traffic": traffic.get("momentum_kernel"),
                    "peak_note": f"measured copy bandwidth ({peaks['source']})"}

    result = {
        "metric": METRIC, "value": round(ms, 4), "unit": "ms", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": _config(args.layers, world),
        "gram_ns": {"ms": round(gram_ms, 4), "tflops": round(tflops, 2),
                    "frac_of_peak": round(tflops / peak_eff, 4),
                    "peak_tflops": round(peak_eff, 1),
                    "flops_bf16": bf, "flops_tf32": tf,
                    "counting": "symmetric products count the upper triangle",
                    "peak_note": f"bf16 {p_bf} ({peaks['source']}, burst) and tf32 = bf16 x "
                                 f"{TF32_RATIO:.3f} (nominal ratio), weighted by flops"},
        "roofline": roofline,
        "roofline_hbm": {"bound": "hbm", "kernel": "momentum_kernel",
                         "achieved": round(mom_gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(mom_gbs / peaks["hbm_gbs"], 4),
                         "frac_of_8tbs": round(mom_gbs / 8000.0, 4),
                         "traffic": traffic.get("momentum_kernel"),
                         "ms_per_step": round(mom_ms, 4),
                         "launches_per_step": mom_launches},
        "matrices_per_s": round(len(mn) / (ms * 1e-3), 1),
        "parts": {nm: {"ms_per_step": round(v, 4)} for nm, v in part_ms.items()},
        "parts_note": "device time of each call, events between the calls inside the same "
                      "full steps (they add up to the step)",
        "kernels": kinds,
        "elementwise": _elementwise(sel_ms, app_ms, own, all_kn, lay, peaks),
        "gpu_launches": int(launches),
        "device_status": st,
    }
    if clocks:
        result["clocks"] = clocks

    if not args.no_e2e:
        result["e2e"] = e2e_measure(args, chunks, step_chunk, exchange_and_update, idx, scale,
                                    barrier, max_over_ranks)

    if world == 1 and not args.no_dion:
        del ws
        torch.cuda.empty_cache()
        result["dion"] = dion_measure(args, Ms, Gs, Ws, mn, dev, peaks)
    if world == 1 and not args.no_sweep:
        torch.cuda.empty_cache()
        result["sweep"] = sweep_points(args, dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


DION_BYTES_PER_ELEM = 30  # B = M + G (10), two reads of B (8), M update (8), bf16 W (4)


def _timed(fn, steps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _dion_line(ms, elems, rank, peaks):
    """ms, and the step's fraction of its HBM and tf32 bounds."""
    gbs = DION_BYTES_PER_ELEM * elems / (ms * 1e-3) / 1e9
    tfl = 8.0 * elems * rank / (ms * 1e-3) / 1e12
    p_tf = peaks["bf16_tflops"] * TF32_RATIO
    return {"ms": round(ms, 4), "hbm_gbs": round(gbs, 1),
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "tflops_tf32": round(tfl, 1), "frac_tf32": round(tfl / p_tf, 4),
            "hbm_bound_ms": round(DION_BYTES_PER_ELEM * elems / (peaks["hbm_gbs"] * 1e9) * 1e3, 4)}


def dion_measure(args, Ms, Gs, Ws, mn, dev, peaks):
    """Dion / Orth-Dion steps at rank 256: one 4096 x 4096 matrix (bf16
    low-rank(64) + noise gradient), and the whole 8B-shaped parameter set in
    one grouped call (the step's buffers, one block per shape; right factors
    one block per weight shape).  Device time per step after warm-up;
    fractions against the algorithmic HBM bytes (30 per element) and the
    tf32 flops (8 m n r)."""
    import torch
    import orthonormalized_update_optimizers_b200 as ouo
    from orthonormalized_update_optimizers_b200 import synth
    K, W = max(3, min(args.steps, 5)), max(3, args.warmup)
    r = 256
    out = {"rank": r, "bytes_per_element": DION_BYTES_PER_ELEM,
           "flops": "8 m n r (tf32)", "peak_note": f"HBM {peaks['hbm_gbs']} GB/s, tf32 = "
           f"bf16 {peaks['bf16_tflops']} x 0.489 ({peaks['source']})"}
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    m = n = 4096
    G = synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(2, 0), torch.bfloat16, dev)
    q0 = torch.linalg.qr(synth.dion_q0(n, r, 1).to(dev))[0].T.contiguous()
    single = {}
    for mode, label in (("colnorm", "dion"), ("qr", "orth_dion")):
        M = torch.zeros(m, n, dtype=torch.float32, device=dev)
        Wt = synth.gaussian((m, n), 5, 0.02, torch.bfloat16, dev)
        Qt = q0.clone()
        p = ouo.dion_params(rank=r, norm_mode=mode)
        wsd = torch.empty(ouo.dion_workspace_bytes([M], p), dtype=torch.uint8, device=dev)
        ms = _timed(lambda: ouo.dion_lowrank_step([M], [G], [Qt], [Wt], p, workspace=wsd,
                                                  status=status), K, W)
        single[label] = _dion_line(ms, m * n, r, peaks)
        del M, Wt, Qt, wsd
    out["matrix_4096x4096"] = single
    # the 8B-shaped set in one call; right factors in one block per shape
    qshapes = {}
    for i, (mm, nn) in enumerate(mn):
        qshapes.setdefault((mm, nn), []).append(i)
    Qs = [None] * len(mn)
    for (mm, nn), members in qshapes.items():
        blk = torch.empty((len(members), r, nn), dtype=torch.float32, device=dev)
        for k, i in enumerate(members):
            blk[k].copy_(q0[:, :nn] if nn == n else
                         torch.linalg.qr(synth.dion_q0(nn, r, 1).to(dev))[0].T)
            Qs[i] = blk[k]
    Mb, Gb, Wb, Qb = ouo.MatBatch(Ms), ouo.MatBatch(Gs), ouo.MatBatch(Ws), ouo.MatBatch(Qs)
    elems = sum(a * b for a, b in mn)
    scales = [math.sqrt(max(1.0, a / b)) for a, b in mn]
    grouped = {}
    for mode, label in (("colnorm", "dion"), ("qr", "orth_dion")):
        p = ouo.dion_params(rank=r, norm_mode=mode)
        need = ouo.dion_workspace_bytes(Mb, p)
        free = torch.cuda.mem_get_info()[0]
        if need > free - (2 << 30):
            grouped[label] = {"skipped": f"workspace {need} B, {free} B free"}
            continue
        wsd = torch.empty(need, dtype=torch.uint8, device=dev)
        ms = _timed(lambda: ouo.dion_lowrank_step(Mb, Gb, Qb, Wb, p, scale=scales,
                                                  workspace=wsd, status=status),
                    max(2, K - 2), 2)
        grouped[label] = dict(_dion_line(ms, elems, r, peaks), workspace_bytes=need)
        del wsd
        torch.cuda.empty_cache()
    out["llama8b_set_grouped"] = dict(grouped, matrices=len(mn), params=elems)
    out["device_status"] = int(status.item())
    return out


def sweep_points(args, dev, peaks):
    """Standard vs Gram Newton-Schulz at the crossover shapes of the sweep
    (m = 1024, n / m = 1, 4, 16; bf16 low-rank(64) + noise, normalization
    on, 5 iterations, one batch of about 2^29 elements per shape).  The
    full sweep is ``--sweep``."""
    import torch
    import orthonormalized_update_optimizers_b200 as ouo
    from orthonormalized_update_optimizers_b200 import synth
    K, W = max(3, min(args.steps, 5)), max(3, args.warmup)
    p_bf = peaks["bf16_tflops"]
    p_tf = p_bf * TF32_RATIO
    rows = []
    for m, n in ((1024, 1024), (1024, 4096), (1024, 16384)):
        nb = max(1, min(64, (1 << 29) // (m * n)))
        X = ouo.batch_empty([(m, n)] * nb, torch.bfloat16, dev)
        for i in range(nb):
            X[i].copy_(synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, 100 * i + n // m),
                                                torch.bfloat16, dev))
        O = [torch.empty_like(x) for x in X]
        Xb, Ob = ouo.MatBatch(X), ouo.MatBatch(O)
        row = {"m": m, "n": n, "batch": nb}
        kk = min(m, n)
        std_tf = ITERS * kk * kk * (kk + 1)
        std_bf = std_ns_flops(m, n) - std_tf
        gbf, gtf = gram_ns_flops(m, n)
        for name, fn_name, bf, tf in (("standard", "ns_orthogonalize", std_bf, std_tf),
                                      ("gram", "gram_ns_orthogonalize", gbf, gtf)):
            params = ouo.ns_params()
            wsb = getattr(ouo, fn_name.replace("orthogonalize", "workspace_bytes"))(Xb, params)
            wsn = torch.empty(wsb, dtype=torch.uint8, device=dev)
            fn = getattr(ouo, fn_name)
            ms = _timed(lambda: fn(Xb, Ob, params, workspace=wsn), K, W)
            tfl = nb * (bf + tf) / (ms * 1e-3) / 1e12
            pk = (bf + tf) / (bf / p_bf + tf / p_tf)
            row[name] = {"ms": round(ms, 4), "tflops": round(tfl, 1),
                         "frac_of_peak": round(tfl / pk, 4)}
            del wsn
        row["gram_speedup"] = round(row["standard"]["ms"] / row["gram"]["ms"], 3)
        rows.append(row)
        del X, O, Xb, Ob
        torch.cuda.empty_cache()
    return {"points": rows, "peak_note": f"bf16 {p_bf} ({peaks['source']}, burst), tf32 = "
            "bf16 x 0.489, weighted by each point's bf16 / tf32 flops"}


def _elementwise(sel_ms, app_ms, own, all_kn, lay, peaks):
    """HBM figures of the selection + gather and weight-update kernels:
    gather reads B[S] (fp32) and writes X0 (bf16) and M[S] (fp32), 10 bytes
    per kept element; the update reads and writes W[S] (bf16) and reads O
    (bf16), 6 bytes per kept element (every rank updates all matrices)."""
    kept_own = sum(all_kn[i][0] * all_kn[i][1] for i in own)
    kept_all = sum(k * n for k, n in all_kn)
    out = {}
    for name, ms, nbytes in (("select_gather", sel_ms, 10 * kept_own),
                             ("apply_update", app_ms, 6 * kept_all)):
        gbs = nbytes / (ms * 1e-3) / 1e9 if ms > 0 else 0.0
        out[name] = {"ms_per_step": round(ms, 4), "bytes_per_step": nbytes,
                     "achieved_gbs": round(gbs, 1),
                     "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4),
                     "frac_of_8tbs": round(gbs / 8000.0, 4)}
    return out


def e2e_measure(args, chunks, step_chunk, exchange_and_update, idx, scale, barrier,
                max_over_ranks):
    """The same step through the public API with the gradients arriving from
    pinned host memory each step and the step's result (kept-row indices and
    per-matrix scales) read back to the host.  The step runs in chunks of
    layers: chunk c+1's gradients are copied on a second stream while chunk c
    is stepped, then the updates are exchanged and applied."""
    import torch
    Gs = [g for ch in chunks for g in ch["G"]]
    total = sum(g.numel() for g in Gs)
    host = torch.empty(max(1, total), dtype=torch.bfloat16, pin_memory=True)
    views, off = [], 0
    for g in Gs:
        v = host[off:off + g.numel()].view(g.shape)
        v.copy_(g)
        views.append(v)
        off += g.numel()
    hviews, pos = [], 0
    for ch in chunks:
        hviews.append(views[pos:pos + len(ch["G"])])
        pos += len(ch["G"])
    idx_h = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
    sc_h = torch.empty(scale.shape, dtype=scale.dtype, pin_memory=True)
    main = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    steps = max(1, min(args.steps, 5))

    def one_step():
        # chunk c's gradients may be overwritten only after the previous
        # step's chunk c has been stepped
        copy.wait_stream(main)
        done = []
        for ch, hv in zip(chunks, hviews):
            with torch.cuda.stream(copy):
                for g, v in zip(ch["G"], hv):
                    g.copy_(v, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy)
            done.append(ev)
        for ch, ev in zip(chunks, done):
            main.wait_event(ev)
            step_chunk(ch)
        exchange_and_update()
        idx_h.copy_(idx, non_blocking=True)
        sc_h.copy_(scale, non_blocking=True)

    one_step()  # warm-up of the chunked schedule
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one_step()
    e1.record()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps)
    return {"value": round(ms, 3), "unit": "ms", "steps": steps,
            "h2d_bytes_per_step": total * 2,
            "d2h_bytes_per_step": idx.numel() * 4 + scale.numel() * 4,
            "schedule": f"gradients copied in chunks of {CHUNK_LAYERS} layers on a copy "
                        "stream, overlapped with the previous chunk's step"}


def run_sweep(args):
    """Standard vs Gram Newton-Schulz over square-to-wide shapes (bf16
    low-rank(64) + noise inputs, normalization on, one batch per shape sized
    to about 2^29 elements), and Dion / Orth-Dion steps on one 4096 x 4096
    matrix over the rank.  Device time per call with CUDA events after
    warm-up; prints one JSON line."""
    import torch

    import orthonormalized_update_optimizers_b200 as ouo
    from orthonormalized_update_optimizers_b200 import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    K, W = max(args.steps, 1), max(args.warmup, 3)

    def timed(fn):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    peaks = _peaks()
    p_bf = peaks["bf16_tflops"]
    p_tf = p_bf * TF32_RATIO

    def peak_for(bf, tf):
        return (bf + tf) / (bf / p_bf + tf / p_tf)

    sampler = ClockSampler(0)
    sampler.start()
    ns_rows = []
    for m in (512, 1024, 2048, 4096, 8192):
        for ratio in (1, 4, 16):
            n = m * ratio
            nb = max(1, min(64, (1 << 29) // (m * n)))
            X = [synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, 100 * i + ratio),
                                          torch.bfloat16, dev) for i in range(nb)]
            O = [torch.empty_like(x) for x in X]
            Xb, Ob = ouo.MatBatch(X), ouo.MatBatch(O)
            row = {"m": m, "n": n, "batch": nb}
            kk = min(m, n)
            std_tf = ITERS * kk * kk * (kk + 1)
            std_bf = std_ns_flops(m, n) - std_tf
            gbf, gtf = gram_ns_flops(m, n)
            for name, fn_name, flops, pk in (
                    ("standard", "ns_orthogonalize", std_bf + std_tf, peak_for(std_bf, std_tf)),
                    ("gram", "gram_ns_orthogonalize", gbf + gtf, peak_for(gbf, gtf))):
                params = ouo.ns_params()
                wsb = getattr(ouo, fn_name.replace("orthogonalize", "workspace_bytes"))(Xb, params)
                ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
                fn = getattr(ouo, fn_name)
                ms = timed(lambda: fn(Xb, Ob, params, workspace=ws))
                tfl = nb * flops / ms / 1e9
                row[name] = {"ms": round(ms, 4), "tflops": round(tfl, 1),
                             "frac_of_peak": round(tfl / pk, 4),
                             "matrices_per_s": round(nb / (ms * 1e-3), 1),
                             "us_per_matrix": round(ms * 1e3 / nb, 2)}
                del ws
            row["gram_speedup"] = round(row["standard"]["ms"] / row["gram"]["ms"], 3)
            ns_rows.append(row)
            del X, O, Xb, Ob
            torch.cuda.empty_cache()

    dion_rows = []
    m = n = 4096
    G = synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, 7), torch.bfloat16, dev)
    for r in (64, 128, 256, 512, 1024):
        for mode in ("colnorm", "qr"):
            M = torch.zeros(m, n, dtype=torch.float32, device=dev)
            Wt = torch.zeros(m, n, dtype=torch.bfloat16, device=dev)
            q = torch.linalg.qr(synth.dion_q0(n, r, 1).to(dev))[0]
            Qt = q.T.contiguous()
            p = ouo.dion_params(rank=r, norm_mode=mode)
            ws = torch.empty(ouo.dion_workspace_bytes([M], p), dtype=torch.uint8, device=dev)
            status = torch.zeros(1, dtype=torch.int32, device=dev)
            ms = timed(lambda: ouo.dion_lowrank_step([M], [G], [Qt], [Wt], p,
                                                      workspace=ws, status=status))
            gemm = 8 * m * n * r
            dion_rows.append({"r": r, "mode": mode, "ms": round(ms, 4),
                              "gemm_tflops": round(gemm / ms / 1e9, 1),
                              "status": int(status.item())})
            del M, Wt, Qt, ws
    clocks = sampler.stop()
    print(json.dumps({"mode": "sweep", "unit": "ms per call (device time)", "steps": K,
                      "peak_note": f"frac_of_peak: against bf16 {p_bf} TFLOP/s ({peaks['source']}, "
                                   f"burst) and tf32 = bf16 x {TF32_RATIO:.3f}, weighted by each "
                                   "point's bf16 / tf32 flops",
                      "warmup": W, "dtype": "bf16 (k x k products tf32; Dion tf32)",
                      "data": "synthetic low-rank(64) + N(0, 0.02^2) noise",
                      "ns": ns_rows, "dion": dion_rows, "clocks": clocks}), flush=True)


def run_micro(args):
    """One kernel-level case (for ncu captures): W warm-up calls, then K
    calls timed with CUDA events; prints one JSON line."""
    import torch

    import orthonormalized_update_optimizers_b200 as ouo
    from orthonormalized_update_optimizers_b200 import synth

    dev = torch.device("cuda", 0)
    m, n = args.m, args.n
    if args.micro == "gram":
        X = [synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, 500 + i),
                                      torch.bfloat16, dev) for i in range(args.nb)]
        O = [torch.empty_like(x) for x in X]
        Xb, Ob = ouo.MatBatch(X), ouo.MatBatch(O)
        p = ouo.ns_params()
        ws = torch.empty(ouo.gram_ns_workspace_bytes(Xb, p), dtype=torch.uint8, device=dev)
        fn = lambda: ouo.gram_ns_orthogonalize(Xb, Ob, p, workspace=ws)  # noqa: E731
        flops = args.nb * sum(gram_ns_flops(m, n))
        case = f"Gram NS, {args.nb} x bf16 {m}x{n}"
    elif args.micro == "dion_set":
        r = args.rank
        shapes = [(a, b) for _, a, b in synth.llama8b_shapes(args.layers)]
        Ms = ouo.batch_empty(shapes, torch.float32, dev)
        Gs = ouo.batch_empty(shapes, torch.bfloat16, dev)
        Ws = ouo.batch_empty(shapes, torch.bfloat16, dev)
        # right factors in one block per weight shape (as the bench line's
        # grouped measurement lays them out), so that every group's Q_state
        # is evenly strided
        qblk = {}
        for i, (a, b) in enumerate(shapes):
            qblk.setdefault((a, b), []).append(i)
        Qs = [None] * len(shapes)
        for (a, b), members in qblk.items():
            blk = torch.empty((len(members), r, b), dtype=torch.float32, device=dev)
            for k, i in enumerate(members):
                Qs[i] = blk[k]
        q0 = {}
        for i, (a, b) in enumerate(shapes):
            Gs[i].copy_(synth.lowrank_plus_noise(a, b, 64, 0.02, synth.seed_for(4, 100 + i),
                                                 torch.bfloat16, dev))
            Ms[i].zero_()
            Ws[i].copy_(synth.gaussian((a, b), synth.seed_for(4, 600 + i), 0.02,
                                       torch.bfloat16, dev))
            if b not in q0:
                q0[b] = torch.linalg.qr(synth.dion_q0(b, r, 1).to(dev))[0].T.contiguous()
            Qs[i].copy_(q0[b])
        Mb, Gb, Wb, Qb = ouo.MatBatch(Ms), ouo.MatBatch(Gs), ouo.MatBatch(Ws), ouo.MatBatch(Qs)
        p = ouo.dion_params(rank=r, norm_mode=args.mode)
        scales = [math.sqrt(max(1.0, a / b)) for a, b in shapes]
        ws = torch.empty(ouo.dion_workspace_bytes(Mb, p), dtype=torch.uint8, device=dev)
        fn = lambda: ouo.dion_lowrank_step(Mb, Gb, Qb, Wb, p, scale=scales,  # noqa: E731
                                           workspace=ws)
        flops = 8 * r * sum(a * b for a, b in shapes)
        case = (f"{'Orth-Dion' if args.mode == 'qr' else 'Dion'} step, 8B-shaped set, "
                f"{args.layers} layer(s), {len(shapes)} matrices, r={r}")
    else:
        r = args.rank
        G = synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, 7), torch.bfloat16, dev)
        M = torch.zeros(m, n, dtype=torch.float32, device=dev)
        W = torch.zeros(m, n, dtype=torch.bfloat16, device=dev)
        Qt = torch.linalg.qr(synth.dion_q0(n, r, 1).to(dev))[0].T.contiguous()
        p = ouo.dion_params(rank=r, norm_mode=args.mode)
        ws = torch.empty(ouo.dion_workspace_bytes([M], p), dtype=torch.uint8, device=dev)
        fn = lambda: ouo.dion_lowrank_step([M], [G], [Qt], [W], p, workspace=ws)  # noqa: E731
        flops = 8 * m * n * r
        case = f"{'Orth-Dion' if args.mode == 'qr' else 'Dion'} step, {m}x{n}, r={r}"
    for _ in range(max(args.warmup, 1)):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"mode": "micro", "case": case, "ms": round(ms, 4),
                      "tflops": round(flops / ms / 1e9, 1), "steps": args.steps,
                      "warmup": args.warmup}), flush=True)


def main():
    args = _args()
    if args.micro:
        run_micro(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
