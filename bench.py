#!/usr/bin/env python
"""Benchmark: one Muon optimizer step (momentum, Nesterov, Frobenius
normalisation, five quintic Newton-Schulz iterations, update scaling and
decoupled weight decay) over the Kimi-K2-shaped parameter set on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload kimi-k2|dense|dense16|moe|single] [--mode standard|gram|gram_stabilized]
                    [--compute bf16|fp16|fp32]

A step is one muon_step call over all matrices of the workload (inputs resident
in HBM).  The metric is effective TFLOP/s: the iteration's algorithmic FLOPs
(every product 2 * rows * cols * inner, 4 m n^2 + 2 n^3 per standard
iteration, as the Gram Newton-Schulz write-up counts them) divided by the
device time of the step; ms per step is reported beside it.  Multi-GPU runs
(torchrun, one process per GPU) give every rank its own full parameter set
(weak scaling, no collective on the data path); the step time is the max over
ranks.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (one expert matrix per step) on the host cores.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "NS-orthogonalization ms/optimizer-step & effective TFLOP/s (% of bf16 peak)"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense TF32 : BF16 tensor rate on B200

# Sources of each product kernel class: a DRAM-traffic figure holds only for
# the kernel it was captured on, so each entry of MEASURED_TRAFFIC records the
# hash of these files at capture time, and a changed kernel reports null.
KERNEL_SOURCES = {
    "tc_chain": ("gemm_chain.cu", "tc_common.cuh"),
    "tc_product": ("gemm_tc2.cu", "gemm_tc.cu", "tc_common.cuh"),
    "tc_product[symmetric]": ("gemm_tc2.cu", "gemm_tc.cu", "tc_common.cuh"),
    "tc_product[3xtf32]": ("gemm_tf32.cu", "tc_common.cuh"),
}
# (workload, compute type, kernel class) -> (source hash, DRAM bytes read +
# written per launch, averaged over the launches of one step, from an ncu
# launch list of `python bench.py --workload <w> --compute <c> --steps 1
# --warmup 1` with --metrics dram__bytes_read.sum,dram__bytes_write.sum).
MEASURED_TRAFFIC: dict = {
    ("kimi-k2", "fp16", "tc_product"): ("b6ba3e11bb008431", 17.47e9),
    ("kimi-k2", "fp16", "tc_product[symmetric]"): ("b6ba3e11bb008431", 7.03e9),
    # captured on the 16-matrix dense16 set (0.674 GB per launch), x 4 for the
    # 64-matrix dense set: the products' traffic grows with the matrix count
    ("dense", "fp32", "tc_product[3xtf32]"): ("59e49be3ff193377", 2.69e9),
    ("dense16", "fp32", "tc_product[3xtf32]"): ("59e49be3ff193377", 0.674e9),
}
def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=["kimi-k2", "kimi-k2-experts16", "dense", "dense16", "moe", "single"], default="kimi-k2",
                   help="kimi-k2-experts16 / dense16: 16 matrices of the K2 / dense set (small cases for profiling)")
    p.add_argument("--mode", choices=["standard", "gram", "gram_stabilized"], default="standard")
    p.add_argument("--compute", choices=["bf16", "fp16", "fp32"], default=None,
                   help="storage type of the chain (default: the workload's, bf16); fp32 runs 3xTF32 products")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-compare", action="store_true", help="skip the stabilised-Gram comparison run")
    p.add_argument("--workspace-gb", type=float, default=24.0, help="workspace cap (chunks the step beyond it)")
    p.add_argument("--graph", action="store_true",
                   help="replay the step from a CUDA graph (launch-latency-bound workloads such as 'single')")
    p.add_argument("--sharded", action="store_true",
                   help="strong scaling: shard one workload across the ranks (ownership by NS FLOPs, owner "
                        "broadcast of the updated weights) instead of one full workload per rank")
    p.add_argument("--report", choices=["stress", "parity"], default=None,
                   help="stress: the ill-conditioned sweep (one JSON line per (n, alpha) point); parity: errors "
                        "against the fp64 oracle on sampled matrices of each workload, every form")
    return p.parse_args()


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's value (device-side all-reduce MAX); identity on one process."""
    if dist is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Weak scaling: every rank runs the full workload; value = all ranks' FLOPs / max step time."""
    return world * flops_per_rank_step / (ms_per_step / 1e3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def build_workload(name, device):
    import synth
    if name == "kimi-k2":
        w = synth.kimi_k2(device=device)
    elif name == "kimi-k2-experts16":
        w = synth.kimi_k2(device=device, counts=[16, 0, 0, 0])
    elif name == "dense":
        w = synth.dense_projection(device=device)
    elif name == "dense16":  # 16 of the dense matrices: small enough for a full profiler capture
        w = synth.dense_projection(device=device, count=16)
    elif name == "moe":
        w = synth.moe_layer(device=device)
    else:
        w = synth.single_fp32(device=device)
    params, grads, moms = [], [], []
    for g in w.groups:
        params += g.W
        grads += g.G
        moms += g.M
    return w, params, grads, moms


def workload_config(w, params, mode, steps_note):
    shapes = {}
    for p in params:
        k = "x".join(map(str, p.shape))
        shapes[k] = shapes.get(k, 0) + 1
    return {"workload": w.name, "matrices": len(params), "shapes": shapes, "mode": mode,
            "ns_iters": 5, "coeffs": [3.4445, -4.7750, 2.0315], "momentum": 0.95, "nesterov": True, "lr": 0.02,
            "weight_decay": 0.1, "scale_coef": 0.2, "l2": steps_note}


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling during the timed region."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,clocks.mem")

    def __init__(self, device):
        self.uuid = None
        try:
            u = str(torch.cuda.get_device_properties(device).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
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
        self.file.flush()
        rows = []
        for line in open(self.file.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and parts[0] != self.uuid:
                continue
            rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        sm = [num(r[1]) for r in rows]
        mx = max(num(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        mem = [num(r[9]) for r in rows if len(r) > 9]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(num(r[3]) for r in rows),
                "mem_mhz": statistics.median(mem) if mem else None}


def kernel_source_hash(kernel: str) -> str | None:
    import hashlib
    files = KERNEL_SOURCES.get(kernel)
    if not files:
        return None
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "newton_schulz_matrix_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload, compute, kernel):
    """Captured DRAM bytes per launch, or None when there is no capture of the
    current kernel source for this workload."""
    e = MEASURED_TRAFFIC.get((workload, compute, kernel))
    if e is None or e[0] != kernel_source_hash(kernel):
        return None
    return e[1]


def roofline_from_profile(prof, peaks, peak_kind, workload=None, compute="fp16"):
    """Roofline of the dominant product kernel class (the one with the most
    device time), from the library's per-launch profile.

    achieved = FLOPs the tensor cores execute in that class (whole tiles; the
    upper-triangle tiles of symmetric products; three TF32 MMAs per 3xTF32
    product) / its device time, against the tensor peak for its input type:
    the sustained bf16 peak for 16-bit products (they run inside a seconds-long
    stream of steps under the power cap; fp16 and bf16 share the kind::f16
    rate), the burst bf16 peak x the nominal TF32:BF16 ratio for 3xTF32
    (those steps run at the maximum clock).  The algorithmic rate (2 M N K per
    product) is given beside it; every class is listed under by_kernel."""
    fp32 = compute == "fp32"
    bf16_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    tf32_peak = round(peaks["bf16_tflops"] * TF32_PER_BF16, 1)
    hbm = peaks["hbm_gbs"]
    rows = []
    for r in prof:
        k = r["kernel"]
        if r["ms"] <= 0:
            continue
        sec = r["ms"] / 1e3
        row = {"kernel": k, "launches": r["launches"], "ms": round(r["ms"], 4)}
        if k.startswith("tc_"):
            peak = tf32_peak if k.endswith("[3xtf32]") else bf16_sust
            ex = r.get("exec_flops", r["flops"])
            row.update(bound="tensor", executed_tflops=round(ex / sec / 1e12, 1),
                       algorithmic_tflops=round(r["flops"] / sec / 1e12, 1), peak=peak,
                       frac=round(ex / sec / 1e12 / peak, 4), exec_flops_per_launch=ex / r["launches"])
        elif r["bytes"] > 0:
            row.update(bound="hbm", gbs=round(r["bytes"] / sec / 1e9, 1), peak=hbm,
                       frac=round(r["bytes"] / sec / 1e9 / hbm, 4))
        rows.append(row)
    tensor = [x for x in rows if x.get("bound") == "tensor" and x["kernel"].endswith("[3xtf32]") == fp32]
    if not tensor:
        return None
    dom = max(tensor, key=lambda x: x["ms"])
    peak_source = (f"{peak_kind} bf16_tflops (burst) x {TF32_PER_BF16:.4f} (nominal TF32:BF16)" if fp32 else
                   f"{peak_kind} bf16_tflops_sustained (kernel timed inside a long step)")
    return {"bound": "tensor", "kernel": dom["kernel"],
            "achieved": dom["executed_tflops"], "peak": dom["peak"], "unit": "TFLOP/s", "frac": dom["frac"],
            "achieved_is": "executed tensor-core FLOPs / device time (CUDA events around each launch)",
            "peak_source": peak_source, "algorithmic_tflops": dom["algorithmic_tflops"],
            "per_launch_ms": round(dom["ms"] / dom["launches"], 4),
            "per_launch_exec_flops": dom["exec_flops_per_launch"],
            "traffic": measured_traffic(workload, compute, dom["kernel"]),
            "traffic_note": "dram__bytes_read.sum + dram__bytes_write.sum per launch (ncu launch list of the "
                            "same workload and kernel source); null when no capture of this source exists",
            "by_kernel": rows}


def cpu_baseline_sample(w, hp, budget_s=20.0):
    """Time the fp64 oracle on whole expert matrices until ~budget_s of CPU work."""
    import numpy as np
    import oracle
    from threadpoolctl import threadpool_info
    g = w.groups[0]
    done_flops = 0.0
    t0 = time.perf_counter()
    n = 0
    while n < len(g.W):
        W = g.W[n].double().cpu().numpy()
        G = g.G[n].double().cpu().numpy()
        M = g.M[n].double().cpu().numpy()
        ts = time.perf_counter()
        oracle.muon_step(W, G, M, lr=hp["lr"], momentum=hp["momentum"], nesterov=hp["nesterov"],
                         weight_decay=hp["weight_decay"], scale_coef=hp["scale_coef"], eps=hp["eps"],
                         coeffs=hp["coeffs"], mode=hp["mode"], restart_after=hp["restart_after"])
        done_flops += oracle.flops(g.rows, g.cols, len(hp["coeffs"]), hp["mode"], hp["restart_after"])
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
        del W, G, M, ts
    el = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": done_flops / el / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {len(g.W)} matrices of shape {g.rows}x{g.cols}, full Muon step in fp64 "
                      f"({done_flops / 1e12:.2f} TFLOP in {el:.1f} s)"}


def run_reference(args):
    """--impl reference: the fp64 oracle on the host cores, one matrix per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synth
    from threadpoolctl import threadpool_info
    w = synth.kimi_k2(device="cpu", counts=[1, 0, 0, 0]) if args.workload == "kimi-k2" else build_workload(args.workload, "cpu")[0]
    hp = dict(w.hp, mode=args.mode)
    g = w.groups[0]
    W = g.W[0].double().numpy(); G = g.G[0].double().numpy(); M = g.M[0].double().numpy()
    def one():
        oracle.muon_step(W, G, M, lr=hp["lr"], momentum=hp["momentum"], nesterov=hp["nesterov"],
                         weight_decay=hp["weight_decay"], scale_coef=hp["scale_coef"], eps=hp["eps"],
                         coeffs=hp["coeffs"], mode=hp["mode"], restart_after=hp["restart_after"])
    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = (time.perf_counter() - t0) / max(args.steps, 1)
    fl = oracle.flops(g.rows, g.cols, len(hp["coeffs"]), hp["mode"], hp["restart_after"])
    value = fl / el / 1e12
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    sample = f"one {g.rows}x{g.cols} matrix per step (of the {w.name} set), full Muon step in fp64"
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "mode": hp["mode"], "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def sigma_band_device(U, O, coeffs, eps=1e-7):
    """max |sigma_i(O) - f^K(sigma_i(U)/(||U||_F+eps))| via fp64 Gram eigenvalues on the device."""
    import numpy as np
    def svals(X):
        X = X.double()
        if X.shape[0] > X.shape[1]:
            X = X.T
        return torch.sqrt(torch.linalg.eigvalsh(X @ X.T).clamp_min(0)).cpu().numpy()
    su, so = svals(U), svals(O)
    t = su / (math.sqrt(float(np.sum(su * su))) + eps)
    for a, b, c in coeffs:
        t = a * t + b * t ** 3 + c * t ** 5
    return float(np.max(np.abs(np.sort(so) - np.sort(t))))


def run_stress_report(args):
    """Ill-conditioned sweep: n in {1024, 2048, 4096}, alpha in {1, 2, 4, 8}, 32
    matrices per point with log-uniform singular values in [1e-6, 1]; for each
    form: device time, Inf/NaN count, sigma-band deviation (matrix 0, any size),
    error against the fp64 oracle (matrix 0, n = 1024), FLOPs saved vs standard."""
    import numpy as np
    import newton_schulz_matrix_b200 as nsm
    import synth
    dev = torch.device("cuda", 0)
    q5 = [synth.QUINTIC] * 5
    for n in (1024, 2048, 4096):
        for alpha in (1, 2, 4, 8):
            mats = synth.stress_point(n, alpha, count=32, device=dev)
            std_flops = nsm.muon_ns_flops(n, alpha * n)
            line = {"report": "stress", "n": n, "alpha": alpha, "matrices": 32, "modes": {}}
            for mode in ("standard", "gram", "gram_stabilized"):
                ys = [m.clone() for m in mats]
                ws = torch.empty(nsm.muon_ns_workspace_size(32, n, alpha * n, mode=mode), dtype=torch.uint8, device=dev)
                st = torch.zeros(32, dtype=torch.int32, device=dev)
                nsm.muon_ns_batched(ys, mode=mode, workspace=ws, status=st)
                torch.cuda.synchronize()
                bad = int((st != 0).sum())
                finite0 = bool(torch.isfinite(ys[0]).all())
                band = sigma_band_device(mats[0].float(), ys[0].float(), q5) if finite0 else None
                err = None
                if n == 1024 and finite0:
                    import oracle
                    U = mats[0].double().cpu().numpy()
                    ref = oracle.newton_schulz(U, q5, mode=mode)
                    err = float(np.linalg.norm(ys[0].double().cpu().numpy() - ref) / np.linalg.norm(ref))
                ys2 = [m.clone() for m in mats]
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                nsm.muon_ns_batched(ys2, mode=mode, workspace=ws)
                e0.record()
                for _ in range(3):
                    nsm.muon_ns_batched(ys2, mode=mode, workspace=ws)
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / 3
                fl = nsm.muon_ns_flops(n, alpha * n, mode=mode)
                line["modes"][mode] = {"ms": round(ms, 3), "nonfinite_matrices": bad, "sigma_band_dev": band,
                                       "rel_err_vs_oracle": err, "flops": 32 * fl,
                                       "flops_saved_vs_standard": round(1 - fl / std_flops, 4),
                                       "effective_tflops": round(32 * fl / ms / 1e9, 1)}
                del ys, ys2, ws
            print(json.dumps(line), flush=True)
            del mats
            torch.cuda.empty_cache()


def run_parity_report(args):
    """Errors against the fp64 oracle at the workloads' full sizes: each
    workload runs as one Muon step in the bench's launch configuration (fp32
    copies of W, so that O = (decay W0 - W1) / step is exact), and sampled
    matrices are compared with oracle.muon_step.  One JSON line per (workload,
    form, compute type, matrix): relative Frobenius error, the oracle's
    stored-precision floor for that chain, sigma-band deviation, oracle time."""
    import numpy as np
    import newton_schulz_matrix_b200 as nsm
    import oracle
    import synth
    dev = torch.device("cuda", 0)
    hp = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2, eps=1e-7,
              coeffs=[synth.QUINTIC] * 5)

    def floor_of(U, mode, chain):
        X, _ = oracle.orient(U)
        f = 1.0 / (oracle.frobenius_norm(X) + hp["eps"])
        exact = oracle.ns_standard(X * f, hp["coeffs"]) if mode == "standard" else oracle.ns_gram(
            X * f, hp["coeffs"], 0 if mode == "gram" else 2)
        start, pre = (oracle.round_to(X, "bf16"), f) if chain == "bf16" else (oracle.round_to(X * f, chain), None)
        emu = (oracle.ns_standard_stored(start, hp["coeffs"], chain, prescale=pre) if mode == "standard" else
               oracle.ns_gram_stored(start, hp["coeffs"], chain, 0 if mode == "gram" else 2, prescale=pre))
        return float(np.linalg.norm(emu - exact) / np.linalg.norm(exact)) if np.all(np.isfinite(emu)) else None

    cases = [("dense-64x1024x4096", lambda: synth.dense_projection(device=dev), [0, 1]),
             ("moe-64e", lambda: synth.moe_layer(device=dev), None),
             ("kimi-k2 experts (8 up/gate + 4 down of the set)", lambda: synth.kimi_k2(device=dev, counts=[8, 4, 0, 0]),
              None)]
    for name, make, pick in cases:
        for mode, compute in (("standard", "fp16"), ("standard", "bf16"), ("gram", "fp16"), ("gram_stabilized", "fp16")):
            w = make()
            params, grads, moms, samples = [], [], [], []
            for g in w.groups:
                samples.append(len(params))
                params += [x.float() for x in g.W]
                grads += g.G
                moms += g.M
            if pick is not None:
                samples = pick
            W0 = {i: params[i].double().cpu().numpy() for i in samples}
            M0 = {i: moms[i].double().cpu().numpy() for i in samples}
            step = nsm.MuonStep(params, grads, moms, mode=mode, compute_dtype=compute, **hp)
            step()
            torch.cuda.synchronize()
            status = int((step.status != 0).sum())
            for i in samples:
                r, c = params[i].shape
                G = grads[i].double().cpu().numpy()
                t0 = time.perf_counter()
                Wr, Mr, Or = oracle.muon_step(W0[i], G, M0[i], mode=mode, restart_after=2, **hp)
                oms = (time.perf_counter() - t0) * 1e3
                sc = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
                O = ((1 - hp["lr"] * hp["weight_decay"]) * W0[i] - params[i].double().cpu().numpy()) / sc
                U = oracle.nesterov_blend(G, Mr, hp["momentum"], True)
                err = float(np.linalg.norm(O - Or) / np.linalg.norm(Or))
                chain = compute if mode == "standard" else "fp16"
                band = sigma_band_device(torch.from_numpy(U).to(dev), torch.from_numpy(O).to(dev), hp["coeffs"])
                print(json.dumps({"report": "parity", "workload": name, "mode": mode, "compute": compute,
                                  "shape": [r, c], "rel_err": err, "floor": floor_of(U, mode, chain),
                                  "sigma_band_dev": band, "status_nonzero": status,
                                  "oracle_ms": round(oms, 1)}), flush=True)
            del step, params, grads, moms, w
            torch.cuda.empty_cache()


def main():
    args = parse_args()
    if args.report == "stress":
        run_stress_report(args)
        return
    if args.report == "parity":
        run_parity_report(args)
        return
    if args.impl == "reference":
        run_reference(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1 or (args.sharded and "MASTER_ADDR" in os.environ):
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    import newton_schulz_matrix_b200 as nsm
    peaks, peak_kind = load_peaks()
    w, params, grads, moms = build_workload(args.workload, device)
    hp = dict(w.hp, mode=args.mode)
    compute = hp.get("compute_dtype", "fp16")
    if args.compute is not None:
        compute = args.compute
    ws_cap = int(args.workspace_gb * (1 << 30))
    step_hp = dict(lr=hp["lr"], momentum=hp["momentum"], nesterov=hp["nesterov"], weight_decay=hp["weight_decay"],
                   scale_coef=hp["scale_coef"], eps=hp["eps"], coeffs=hp["coeffs"], mode=hp["mode"],
                   restart_after=hp["restart_after"], compute_dtype=compute)
    flops_step = sum(nsm.muon_ns_flops(p.shape[0], p.shape[1], coeffs=hp["coeffs"], mode=hp["mode"],
                                       restart_after=hp["restart_after"]) for p in params)
    if args.sharded:
        if dist is None:
            raise SystemExit("--sharded needs torchrun (one process per GPU)")
        from newton_schulz_matrix_b200.distributed import ShardedMuonStep
        owner_moms = {i: m for i, m in enumerate(moms)}
        step = ShardedMuonStep(params, grads, owner_moms, local_step_factory=lambda ps, gs, ms, **h: nsm.MuonStep(
            ps, gs, ms, workspace_bytes=ws_cap, **h), **step_hp)
        flops_step /= world  # whole_job_tflops multiplies by world: the set is processed once in total
    else:
        step = nsm.MuonStep(params, grads, moms, workspace_bytes=ws_cap, **step_hp)
    resident = sum(t.numel() * t.element_size() for t in params + grads + moms)
    stream = torch.cuda.current_stream(device)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    run = step
    graph_launches = None
    if args.graph and not args.sharded:
        nsm.muon_profile_begin()
        step()
        torch.cuda.synchronize(device)
        graph_launches = sum(r["launches"] for r in nsm.muon_profile_end())
        graph = step.capture()
        run = graph.replay
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, device)
    # the same steps again with every library launch bracketed by CUDA events on
    # its stream: per-kernel device time for the roofline and the launch count
    # (a separate pass, so the two events per launch stay out of the headline)
    barrier()
    torch.cuda.synchronize(device)
    nsm.muon_profile_begin()
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        step()  # eager even under --graph: a replay makes no library calls to bracket
    p1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    prof = nsm.muon_profile_end()
    prof_ms = p0.elapsed_time(p1) / args.steps
    status = step.local.status.cpu() if args.sharded and step.local is not None else (
        torch.zeros(1, dtype=torch.int32) if args.sharded else step.status.cpu())
    value = whole_job_tflops(world, flops_step, ms)
    launches_timed = sum(r["launches"] for r in prof) if graph_launches is None else graph_launches * args.steps

    # stabilised Gram comparison on the same matrices (context for the Gram-vs-standard claim)
    compare = None
    if graph_launches is not None:
        del run, graph
    if not args.no_compare and args.mode == "standard" and compute != "fp32" and not args.sharded:
        del step
        torch.cuda.empty_cache()
        st2 = nsm.MuonStep(params, grads, moms, workspace_bytes=ws_cap, lr=hp["lr"], momentum=hp["momentum"],
                           nesterov=hp["nesterov"], weight_decay=hp["weight_decay"], scale_coef=hp["scale_coef"],
                           eps=hp["eps"], coeffs=hp["coeffs"], mode="gram_stabilized", restart_after=2)
        st2()
        torch.cuda.synchronize(device)
        barrier()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nrep = max(2, args.steps // 2)
        c0.record(stream)
        for _ in range(nrep):
            st2()
        c1.record(stream)
        torch.cuda.synchronize(device)
        barrier()
        gms = max_over_ranks(c0.elapsed_time(c1) / nrep, dist, device)
        compare = {"gram_stabilized_ms_per_step": round(gms, 3), "standard_ms_per_step": round(ms, 3),
                   "speedup_vs_standard": round(ms / gms, 3)}
        step = st2

    # end to end through the public API: gradients H2D from pinned host memory,
    # the step, updated weights D2H to pinned host memory, every step
    e2e = None
    # pinned host copies of G and W for every rank on this node must fit comfortably in RAM
    local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    host_need = local_world * sum(t.numel() * t.element_size() for t in grads + params)
    try:
        import psutil
        host_free = psutil.virtual_memory().available
    except Exception:
        host_free = 0
    fits = host_need <= 0.6 * host_free
    if dist is not None:  # every rank must take the same branch (the leg has barriers)
        flag = torch.tensor([1.0 if fits else 0.0], device=device)
        dist.all_reduce(flag, op=dist.ReduceOp.MIN)
        fits = bool(flag.item() > 0.5)
    if not args.no_e2e and not fits:
        e2e = {"value": None, "unit": "TFLOP/s", "skipped": f"pinned host buffers ({host_need / 2**30:.0f} GiB "
               f"for {local_world} ranks) exceed 60% of free host memory ({host_free / 2**30:.0f} GiB)"}
    elif not args.no_e2e and not args.sharded:
        hG = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in grads]
        hW = [torch.empty(p.shape, dtype=p.dtype, pin_memory=True) for p in params]
        for h, g in zip(hG, grads):
            h.copy_(g)
        del step
        torch.cuda.synchronize(device)
        torch.cuda.empty_cache()
        # gradients stream in from pinned host memory and updated weights stream out,
        # slice by slice, overlapped with the orthogonalisation of other slices
        e2e_step = nsm.StreamedMuonStep(params, grads, moms, hG, hW, workspace_bytes=ws_cap, **step_hp)
        e2e_step()
        torch.cuda.synchronize(device)
        barrier()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        x1.record(stream)
        torch.cuda.synchronize(device)
        barrier()
        ems = max_over_ranks(x0.elapsed_time(x1) / args.e2e_steps, dist, device)
        e2e = {"value": whole_job_tflops(world, flops_step, ems), "unit": "TFLOP/s", "ms_per_step": round(ems, 3),
               "h2d_bytes_per_step": sum(g.numel() * g.element_size() for g in grads),
               "d2h_bytes_per_step": sum(p.numel() * p.element_size() for p in params)}
        del hG, hW

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(w, hp)

    if rank == 0:
        roof = roofline_from_profile(prof, peaks, peak_kind, args.workload, compute)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "strong" if args.sharded else "weak",
            "vs_baseline": None, "dtype": {"bf16": "bf16", "fp16": "f16", "fp32": "f32"}[compute],
            "dtype_note": (f"chain storage {compute} (X0, A, B or the Gram matrices between the products; "
                           f"fp32 accumulation); parameters W and gradients G stay in their own types "
                           f"({', '.join(sorted({str(p.dtype).replace('torch.', '') for p in params}))}), "
                           "momentum fp32"),
            "data": "synthetic (seeded recipes of the workload; no datasets)",
            "config": dict(workload_config(w, params, hp["mode"], f"inputs larger than L2 ({resident / 2**30:.1f} GiB resident)"),
                           parallelism=(f"sharded over {world} ranks (owner broadcast)" if args.sharded
                                        else f"{world} replica(s), one full workload per GPU"),
                           cuda_graph=bool(args.graph)),
            "pct_of_bf16_peak": round(100 * value / world / peaks["bf16_tflops"], 2),
            "peaks": {"bf16_tflops": peaks["bf16_tflops"], "bf16_tflops_sustained": peaks.get("bf16_tflops_sustained"),
                      "source": peak_kind},
            "flops_per_step": flops_step,
            "clocks": clk, "e2e": e2e, "gpu_launches": launches_timed, "roofline": roof, "cpu_baseline": cpu,
            "profiled_ms_per_step": round(prof_ms, 3),
            "kernels": [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()} for r in prof],
            "status_nonzero": int((status != 0).sum()),
        }
        if compare:
            line["compare"] = compare
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
