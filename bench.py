"""Benchmark of the triangle multiplicative update on B200 (one JSON line on rank 0).

A step is one pass of the hot path over one batch of synthetic input: the outgoing and
the incoming update (tri_mul_forward twice: K1, the offsets pass, K2 and K3 each) on the
OpenFold-shaped pair workload B=1, N=512, c_z=c_h=128, bf16 z with a ragged padding mask.
`value` is milliseconds per layer (one direction) for the whole job, timed with nothing but
the forwards in the timed region; a second, instrumented pass records CUDA events between
the kernels for the per-kernel breakdown and the roofline. Several GPUs run independent
replicas (weak scaling, no collective on the data path). On one GPU the line also carries
`workloads`: the same two measurements for the other seeded configurations (N=256 with its
tail mask, B=4 N=256 c_z=384, and N=2048 incoming then outgoing).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the only other implementation there is)
on this machine's host cores on the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ms/layer and effective TFLOP/s (fraction of bf16 roofline) for tri-mul at N=512, c_z=128"
WORKLOAD = "bf16_n512_ragged"
WORKLOADS = ("bf16_n512_ragged", "bf16_n256_tail10", "bf16_b4_n256_cz384", "bf16_n2048")
CPU_BASELINE_WORKLOADS = ("bf16_n512_ragged", "bf16_n256_tail10", "bf16_b4_n256_cz384")
# the other configurations timed on one GPU next to the headline (the N=64 fp32 one is launch-bound)
EXTRA_WORKLOADS = ("bf16_n256_tail10", "bf16_b4_n256_cz384", "bf16_n2048")
# oracle timings on the host: (workload, threads) pairs run by default; --cpu-full runs all of
# fp32_n64 ... bf16_b4_n256_cz384 on all threads and on one
CPU_DEFAULT_RUNS = (("fp32_n64", 0), ("bf16_n256_tail10", 0), ("bf16_n512_ragged", 0), ("bf16_b4_n256_cz384", 0),
                    ("bf16_n2048", 0), ("fp32_n64", 1), ("bf16_n256_tail10", 1))
L2_BYTES = 126 * 1024 * 1024
KERNEL_NAMES = ("k1_project_kernel", "k2_contract_kernel", "k3_output_kernel")
KERNEL_SOURCES = {"k1_project_kernel": "k1_project.cu", "k2_contract_kernel": "k2_contract.cu",
                  "k3_output_kernel": "k3_output.cu", "pair_transition_kernel": "transition.cu"}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--out-dtype", choices=("f32", "bf16"), default="f32")
    ap.add_argument("--workload", choices=WORKLOADS, default=WORKLOAD,
                    help="the seeded configuration to time (default: the headline N=512 workload; the "
                         "others are for the per-kernel breakdown at other shapes)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the CPU oracle")
    ap.add_argument("--skip-masked", action="store_true",
                    help="switch mask skipping on (leave out wholly masked tiles; off by default)")
    ap.add_argument("--no-transition", action="store_true", help="skip the pair-transition leg")
    ap.add_argument("--no-torch-context", action="store_true",
                    help="skip timing the eager PyTorch composition of the same math (context only)")
    ap.add_argument("--no-pair-update", action="store_true",
                    help="skip the pair-update leg (outgoing + incoming with residuals, eager and as a CUDA graph)")
    ap.add_argument("--no-workloads", action="store_true", help="skip timing the other seeded configurations")
    ap.add_argument("--cpu-full", action="store_true",
                    help="time the oracle on every CPU configuration on all threads and on one thread")
    ap.add_argument("--cpu-oracle-probe", nargs=2, metavar=("WORKLOAD", "DIRECTION"), default=None,
                    help=argparse.SUPPRESS)   # internal: one oracle layer in a fresh process (OMP_NUM_THREADS set)
    return ap.parse_args()


def valid_work(lengths, c_z, c_h):
    """Flops of one layer counting only the valid residues (the work a length-L problem needs):
    the dense formulas of layer_work with N replaced by each batch element's valid length L_b."""
    total = 0
    for L in lengths:
        f, _ = layer_work(1, int(L), c_z, c_h)
        total += sum(f.values())
    return total


def layer_work(B, N, c_z, c_h, out_bytes=4):
    """Algorithmic flops and HBM bytes of one layer, per kernel (dense over N; masked work counted).

    K1 reads z (bf16) and the mask, writes a and b (fp16); K2 reads a, b and writes x; K3
    reads x, z and the mask and writes out. Weights are negligible and not counted.
    """
    P = B * N * N
    flops = {
        "k1_project_kernel": 2 * P * c_z * 4 * c_h,
        "k2_contract_kernel": 2 * B * c_h * N ** 3,
        "k3_output_kernel": 2 * P * c_z * (c_z + c_h),
    }
    nbytes = {
        "k1_project_kernel": P * (2 * c_z + 2 + 2 * 2 * c_h),
        "k2_contract_kernel": P * 3 * 2 * c_h,
        "k3_output_kernel": P * (2 * c_h + 2 * c_z + 2 + out_bytes * c_z),
    }
    return flops, nbytes


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(kernel: str) -> str:
    csrc = os.path.join(ROOT, "protein_pair_representation_b200", "csrc")
    h = hashlib.sha256()
    for name in (KERNEL_SOURCES[kernel], "sm100.cuh", "kernels.h"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        if rec.get("source_hash") == kernel_source_hash(kernel):
            return float(rec["bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(value_ms, dist=None, device=None):
    """The largest of every rank's elapsed time (the job's time); identity on one rank."""
    if dist is None:
        return float(value_ms)
    import torch
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_layer(max_elapsed_ms, steps, n_dirs, world):
    """Whole-job milliseconds per layer: every rank ran `steps` steps of `n_dirs` layers in
    `max_elapsed_ms` (the slowest rank), so the job processed steps * n_dirs * world layers."""
    return max_elapsed_ms / (steps * n_dirs * world)


def dist_setup(gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}")
    return rank, world, local


def cpu_oracle_layer_ms(inp, directions):
    """Wall-clock ms per layer of the fp64 oracle on this host (all its threads)."""
    import oracle
    times = []
    for d in directions:
        t0 = time.perf_counter()
        oracle.trimul(inp.z, inp.mask, inp.weights, d, inp.eps)
        times.append((time.perf_counter() - t0) * 1e3)
    return statistics.mean(times), oracle.num_threads()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_oracle_probe(workload, direction):
    """One oracle layer of `workload` in this (fresh) process; prints its JSON timing. N = 2048
    runs the sampled mode (the 64 x 64 = 4096 entries the parity tests compare)."""
    import oracle
    import trimul_inputs as ti
    inp = ti.make_config(workload)
    sampled = inp.N > 1024
    if sampled:
        I, J = ti.sample_indices(inp.N, 64, seed=inp.seed)
    t0 = time.perf_counter()
    if sampled:
        oracle.trimul_sampled(inp.z, inp.mask, inp.weights, direction, I, J, inp.eps)
    else:
        oracle.trimul(inp.z, inp.mask, inp.weights, direction, inp.eps)
    print(json.dumps({"ms": (time.perf_counter() - t0) * 1e3, "threads": oracle.num_threads(),
                      "sampled": sampled}), flush=True)


def cpu_oracle_runs(runs):
    """Oracle wall-clock ms per layer for (workload, threads) pairs, each in a fresh process
    (threads 0: all of the host's, else OMP_NUM_THREADS=threads), outgoing direction."""
    out = []
    for workload, threads in runs:
        env = dict(os.environ)
        if threads:
            env["OMP_NUM_THREADS"] = str(threads)
        else:
            env.pop("OMP_NUM_THREADS", None)
        try:
            r = subprocess.run([sys.executable, os.path.abspath(__file__), "--cpu-oracle-probe", workload, "outgoing"],
                               env=env, capture_output=True, text=True, timeout=900, cwd=ROOT)
            rec = json.loads(r.stdout.strip().splitlines()[-1])
            out.append({"workload": workload, "threads": rec["threads"], "ms_per_layer": rec["ms"],
                        "what": "4096 sampled entries (64 rows x 64 columns)" if rec.get("sampled") else "full layer"})
        except Exception as exc:                  # the line must not depend on this leg
            out.append({"workload": workload, "threads": threads or None, "error": f"{type(exc).__name__}: {exc}"})
    return out


def run_reference(args):
    """The oracle on the host cores: each step computes one full layer (directions alternate)."""
    rank, world, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    import trimul_inputs as ti
    if args.workload not in CPU_BASELINE_WORKLOADS:
        print(json.dumps({"impl": "reference", "unavailable": f"a full fp64 oracle layer of {args.workload} "
                                                              f"takes hours on the host cores"}), flush=True)
        return
    inp = ti.make_config(args.workload)
    dirs = ti.CONFIGS[args.workload]["directions"]
    import oracle
    for s in range(args.warmup):
        oracle.trimul(inp.z, inp.mask, inp.weights, dirs[s % 2], inp.eps)
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle.trimul(inp.z, inp.mask, inp.weights, dirs[s % 2], inp.eps)
    total_ms = (time.perf_counter() - t0) * 1e3
    ms_layer = total_ms / max(1, args.steps)
    flops, _ = layer_work(inp.B, inp.N, inp.c_z, inp.c_h)
    sample = (f"one full layer per step ({inp.N}x{inp.N} pairs, c_z={inp.c_z}, c_h={inp.c_h}), "
              f"outgoing and incoming alternating, fp64")
    cores = oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": ms_layer, "unit": "ms/layer", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / max(1, args.steps),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(inp, "f64"),
        "effective_tflops": sum(flops.values()) / (ms_layer * 1e-3) / 1e12,
        "cpu_baseline": {"value": ms_layer, "unit": "ms/layer", "cores": cores, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model(), "nproc": os.cpu_count()},
        "e2e": {"value": ms_layer, "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def pair_update_leg(tm, layer, zs, ms_, n_sets, args, dev):
    """ms per pair update (outgoing then incoming update, each a masked residual; z_mid and
    out in bf16) on this rank's workload, launched eagerly and replayed as one CUDA graph per
    input copy. Inputs cycle through the same L2-defeating copies as the main leg."""
    import torch
    try:
        mids = [torch.empty_like(zs[0]) for _ in range(n_sets)]
        outs = [torch.empty_like(zs[0]) for _ in range(n_sets)]
        graphs = [tm.PairUpdateGraph(zs[i], ms_[i], layer, layer) for i in range(n_sets)]

        def eager(s):
            i = s % n_sets
            tm.pair_update(zs[i], ms_[i], layer, layer, out=outs[i], z_mid=mids[i])

        def graph(s):
            graphs[s % n_sets].launch()

        res = {}
        for name, fn in (("eager_ms", eager), ("graph_ms", graph)):
            for s in range(max(3, args.warmup)):
                fn(s)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for s in range(args.steps):
                fn(s)
            e1.record()
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) / args.steps
        tm.check_device_status()
        for g in graphs:
            g.close()
        res.update({"unit": "ms per pair update (two triangle updates with residuals; one layer handle for both)",
                    "gpu_launches_per_update": 2 * tm.kernels_per_forward()})
        return res
    except Exception as exc:       # the headline line must not depend on this leg
        return {"error": f"{type(exc).__name__}: {exc}"}


def torch_composition(z, mask, w, direction, eps):
    """The same update as a plain eager PyTorch composition (layer_norm, linear, sigmoid,
    einsum): a context figure for the hand-written kernels, not part of the library.
    w holds the layer's sixteen arrays under the ABI names; biases and affines may be None."""
    import torch
    F = torch.nn.functional
    zh = F.layer_norm(z, (z.shape[-1],), w["ln_in_g"], w["ln_in_b"], eps)
    m = 1.0 if mask is None else mask[..., None]
    a = m * torch.sigmoid(F.linear(zh, w["w_ag"], w["b_ag"])) * F.linear(zh, w["w_ap"], w["b_ap"])
    b = m * torch.sigmoid(F.linear(zh, w["w_bg"], w["b_bg"])) * F.linear(zh, w["w_bp"], w["b_bp"])
    if direction == "outgoing":
        x = torch.einsum("bikc,bjkc->bijc", a, b)
    else:
        x = torch.einsum("bkic,bkjc->bijc", a, b)
    xn = F.layer_norm(x, (x.shape[-1],), w["ln_out_g"], w["ln_out_b"], eps)
    return m * torch.sigmoid(F.linear(zh, w["w_g"], w["b_g"])) * F.linear(xn, w["w_o"], w["b_o"])


def torch_composition_leg(zs, ms_, w, eps, dirs, n_sets, args):
    """ms per layer of torch_composition on the same bf16 inputs and weights (cuBLAS GEMMs and
    a batched-GEMM einsum, all eager), timed like the main leg: context, not a target."""
    import torch
    try:
        def step(s):
            for d in dirs:
                torch_composition(zs[s % n_sets], ms_[s % n_sets], w, d, eps)

        for s in range(max(3, args.warmup)):
            step(s)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(args.steps):
            step(s)
        e1.record()
        torch.cuda.synchronize()
        return {"ms_per_layer": e0.elapsed_time(e1) / (args.steps * len(dirs)),
                "what": "eager PyTorch composition of the same math (layer_norm, linear, sigmoid, einsum) "
                        "on the same bf16 inputs; context, not a target"}
    except Exception as exc:       # the headline line must not depend on this leg
        return {"error": f"{type(exc).__name__}: {exc}"}


def transition_leg(tm, zs, ms_, n_sets, args, dev):
    """The fused pair transition (out = z + m (relu(z W1^T + b1) W2^T + b2), c = 128, hidden 256)
    on this rank's pair tensors, bf16 in and out, seeded random weights; per-call ms from CUDA
    events over `steps` calls, inputs cycling through the L2-defeating copies."""
    import numpy as np
    import torch
    try:
        rng = np.random.default_rng(1234)
        mk = lambda *shape, scale: torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(
            dev).to(torch.bfloat16)
        pt = tm.PairTransition(mk(256, 128, scale=128 ** -0.5), mk(128, 256, scale=256 ** -0.5),
                               mk(256, scale=0.1), mk(128, scale=0.1))
        outs = [torch.empty_like(zs[0]) for _ in range(n_sets)]
        for s_ in range(max(3, args.warmup)):
            pt.forward(zs[s_ % n_sets], ms_[s_ % n_sets], out=outs[s_ % n_sets])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s_ in range(args.steps):
            pt.forward(zs[s_ % n_sets], ms_[s_ % n_sets], out=outs[s_ % n_sets])
        e1.record()
        torch.cuda.synchronize()
        tm.check_device_status()
        ms = e0.elapsed_time(e1) / args.steps
        P = zs[0].shape[0] * zs[0].shape[1] * zs[0].shape[2]
        c, hidden = pt.c, pt.hidden
        nbytes = P * (2 * c + 2 + 2 * c)               # z in, mask, out (bf16)
        flops = P * 2 * 2 * c * hidden
        peaks = measured_peaks()
        gbs, tfs = nbytes / (ms * 1e-3) / 1e9, flops / (ms * 1e-3) / 1e12
        pt.close()
        return {"ms": ms, "GB_s": gbs, "TFLOP_s": tfs, "hbm_frac": gbs / peaks["hbm_gbs"],
                "tensor_frac": tfs / peaks["bf16_tflops"], "bytes": nbytes, "flops": flops,
                "traffic": recorded_traffic("pair_transition_kernel"),
                "shape": f"c={c}, hidden={hidden}, bf16 in/out, fp16 hidden activation on chip"}
    except Exception as exc:       # the headline line must not depend on this leg
        return {"error": f"{type(exc).__name__}: {exc}"}


def workload_config(inp, compute):
    lengths = [int(v) for v in inp.lengths]
    mask = "all-ones mask" if min(lengths) == inp.N else f"ragged mask (L={lengths if inp.B > 1 else lengths[0]})"
    return {"workload": f"triangle multiplicative update, B={inp.B} N={inp.N} c_z={inp.c_z} c_h={inp.c_h}, "
                        f"bf16 z and weights, {mask}, outgoing + incoming",
            "B": inp.B, "N": inp.N, "c_z": inp.c_z, "c_h": inp.c_h,
            "valid_length": lengths[0] if inp.B == 1 else lengths,
            "directions": ["outgoing", "incoming"], "compute": compute}


class Workload:
    """One seeded configuration on this rank's GPU: inputs (cycled through enough copies that
    every step reads z and the mask from outside L2), the layer with its workspace, outputs."""

    def __init__(self, tm, name, seed, dev, out_dt, skip_masked):
        import numpy as np
        import torch

        import trimul_inputs as ti
        self.name = name
        self.inp = inp = ti.make_config(name, seed=seed)
        self.dirs = ti.CONFIGS[name]["directions"]
        self.z0 = torch.from_numpy(inp.z).to(dev).to(torch.bfloat16)
        self.m0 = torch.from_numpy(inp.mask).to(dev).to(torch.bfloat16)
        self.w = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev).to(torch.bfloat16) for k, v in inp.weights.items()}
        self.layer = tm.TriMulLayer(self.w, eps=inp.eps)
        self.layer.ensure_workspace(inp.B, inp.N, torch.bfloat16)
        if skip_masked:
            self.layer.set_mask_skipping(True)
        self.set_bytes = self.z0.numel() * 2 + self.m0.numel() * 2
        # one copy when it alone is over twice the L2, else enough copies to be
        self.n_sets = 1 if self.set_bytes >= 2 * L2_BYTES else max(2, -(-2 * L2_BYTES // self.set_bytes))
        self.zs = [self.z0] + [self.z0.clone() for _ in range(self.n_sets - 1)]
        self.ms = [self.m0] + [self.m0.clone() for _ in range(self.n_sets - 1)]
        self.outs = [torch.empty(self.z0.shape, dtype=out_dt, device=dev) for _ in self.dirs]
        self.out_bytes = 4 if out_dt == torch.float32 else 2

    def step(self, s, evs=None):
        for di, d in enumerate(self.dirs):
            if evs is not None:
                self.layer.set_timing_events(evs[di])
            self.layer.forward(self.zs[s % self.n_sets], self.ms[s % self.n_sets], d, out=self.outs[di])
        if evs is not None:
            self.layer.set_timing_events(None)

    def l2_note(self):
        if self.n_sets == 1:
            return f"z and mask ({self.set_bytes / 2**20:.0f} MiB) larger than twice the 126 MiB L2"
        return f"z and mask cycle through {self.n_sets} copies ({self.n_sets * self.set_bytes / 2**20:.0f} MiB > 126 MiB L2)"


def time_steps(wl, steps, first, sync_all, dist=None, dev=None, instrumented=False):
    """Device ms of `steps` steps (CUDA events on the launching stream, barrier + synchronize on
    both sides, max over ranks) and, when instrumented, the per-kernel mean ms from the four
    events each forward records between its kernels."""
    import torch
    kev = None
    if instrumented:
        kev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in wl.dirs] for _ in range(steps)]
        for ev in kev:                   # torch creates the CUDA event on first record
            for row in ev:
                for e in row:
                    e.record()
        torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all()
    t0.record()
    for s in range(steps):
        wl.step(first + s, kev[s] if instrumented else None)
    t1.record()
    sync_all()
    elapsed = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    kernel_ms = None
    if instrumented:
        kernel_ms = {k: statistics.mean(ev[d][i].elapsed_time(ev[d][i + 1]) for ev in kev for d in range(len(wl.dirs)))
                     for i, k in enumerate(KERNEL_NAMES)}
    return elapsed, kernel_ms


def bf16_out_pass(tm, wl, steps, sync_all, peaks):
    """The same steps with `out` in z's dtype (bf16) instead of fp32: ms per layer and K3 alone
    with 2-byte output, and the layer's roofline fraction at those bytes. (The headline keeps fp32
    out: a bf16 out alone rounds values near 10x RMS by up to half an ulp, about 0.03 RMS.)"""
    import torch
    saved, saved_bytes = wl.outs, wl.out_bytes
    wl.outs = [torch.empty(wl.z0.shape, dtype=torch.bfloat16, device=wl.z0.device) for _ in wl.dirs]
    wl.out_bytes = 2
    try:
        for s_ in range(3):
            wl.step(s_)
        el, _ = time_steps(wl, steps, 0, sync_all)
        alone = stage_times(tm, wl, steps, sync_all)
        kernels, _, t_ideal = kernel_record(wl.inp, alone, peaks, 2)
        layer_ms = el / (steps * len(wl.dirs))
        return {"ms_per_layer": layer_ms, "layer_roofline_frac": t_ideal / (layer_ms * 1e-3),
                "k3_output_kernel": kernels["k3_output_kernel"]}
    finally:
        wl.outs, wl.out_bytes = saved, saved_bytes


def warm_l2_pass(wl, steps, sync_all):
    """The headline steps with the same z and mask every step (labelled warm L2: at N <= 512 the
    inputs, and part of the intermediates, stay in the 126 MiB L2 between steps)."""
    saved = wl.n_sets
    wl.n_sets = 1
    try:
        for s_ in range(3):
            wl.step(s_)
        el, _ = time_steps(wl, steps, 0, sync_all)
    finally:
        wl.n_sets = saved
    return {"ms_per_layer": el / (steps * len(wl.dirs)), "what": "warm L2: the same inputs every step"}


def valid_length_pass(tm, wl, steps, sync_all):
    """The headline steps with the layer told the mask's valid lengths: the library's rule
    decides whether skipping pays (it does when it leaves out at least 15% of the dense
    flops); ms per layer and that decision."""
    lengths = [int(v) for v in wl.inp.lengths]
    chosen = wl.layer.set_valid_lengths(lengths, wl.inp.N)
    try:
        for s in range(3):
            wl.step(s)
        el, _ = time_steps(wl, steps, 0, sync_all)
    finally:
        wl.layer.set_valid_lengths(None)
    return {"ms_per_layer": el / (steps * len(wl.dirs)), "skipping_chosen": chosen,
            "dense_share_left_out": tm.skip_saving(lengths, wl.inp.N, wl.inp.c_z, wl.inp.c_h)}


def stage_times(tm, wl, steps, sync_all):
    """Each kernel alone: `steps` back-to-back launches of its stage entry point (K1
    tri_mul_project, K2 tri_mul_contract in both directions in turn, K3 tri_mul_output_gate)
    between two CUDA events on the launching stream, every input cycling through copies that
    together exceed twice the L2; mean ms per launch. Successive launches overlap launch and
    prologue with the previous kernel's tail through programmatic dependent launch, as the
    kernels of a forward do. K1 alone does not gather the channel sums of the stored-x offset
    (first 8 pairs of every 64-pair tile), and K2 alone subtracts no offset."""
    import torch
    inp = wl.inp
    shape = (inp.B, inp.c_h, inp.N, inp.N)
    plane = inp.B * inp.c_h * inp.N * inp.N * 2
    n_ab = max(2, -(-2 * L2_BYTES // (2 * plane)))
    n_x = max(2, -(-2 * L2_BYTES // plane))
    dev = wl.z0.device
    A = [torch.empty(shape, dtype=torch.float16, device=dev) for _ in range(n_ab)]
    Bp = [torch.empty(shape, dtype=torch.float16, device=dev) for _ in range(n_ab)]
    X = [torch.empty(shape, dtype=torch.float16, device=dev) for _ in range(n_x)]
    scale = tm.contract_scale(inp.N)
    dirs = wl.dirs
    launch = {
        "k1_project_kernel": lambda s: wl.layer.project(wl.zs[s % wl.n_sets], wl.ms[s % wl.n_sets],
                                                        a=A[s % n_ab], b=Bp[s % n_ab]),
        "k2_contract_kernel": lambda s: tm.contract(A[s % n_ab], Bp[s % n_ab], dirs[s % len(dirs)],
                                                    out=X[s % n_x], x_scale=scale),
        "k3_output_kernel": lambda s: wl.layer.output_gate(wl.zs[s % wl.n_sets], X[s % n_x], wl.ms[s % wl.n_sets],
                                                           out=wl.outs[0], x_scale=scale),
    }
    out = {}
    for k in KERNEL_NAMES:
        for s in range(max(3, n_ab, n_x, wl.n_sets)):
            launch[k](s)
        sync_all()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(steps):
            launch[k](s)
        e1.record()
        sync_all()
        out[k] = e0.elapsed_time(e1) / steps
    del A, Bp, X
    torch.cuda.empty_cache()
    return out


def kernel_record(inp, kernel_ms, peaks, out_bytes, in_step_ms=None):
    """Per-kernel figures from `kernel_ms` (each kernel timed alone); `in_step_ms`, the means of
    the event intervals inside the instrumented steps, is reported beside them."""
    flops, nbytes = layer_work(inp.B, inp.N, inp.c_z, inp.c_h, out_bytes)
    kernels = {}
    for k in KERNEL_NAMES:
        t = kernel_ms[k] * 1e-3
        t_hbm = nbytes[k] / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops[k] / (peaks["bf16_tflops"] * 1e12)
        kernels[k] = {"ms": kernel_ms[k], "GB_s": nbytes[k] / t / 1e9, "TFLOP_s": flops[k] / t / 1e12,
                      "hbm_frac": nbytes[k] / t / 1e9 / peaks["hbm_gbs"],
                      "tensor_frac": flops[k] / t / 1e12 / peaks["bf16_tflops"],
                      "bound": "hbm" if t_hbm >= t_tc else "tensor", "roofline_frac": max(t_hbm, t_tc) / t,
                      "bytes": nbytes[k], "flops": flops[k]}
        if in_step_ms is not None:
            kernels[k]["in_step_ms"] = in_step_ms[k]
    t_ideal = sum(max(nbytes[k] / (peaks["hbm_gbs"] * 1e9), flops[k] / (peaks["bf16_tflops"] * 1e12))
                  for k in KERNEL_NAMES)
    return kernels, flops, t_ideal


def workload_summary(wl, layer_ms, kernel_ms, instr_layer_ms, peaks, in_step_ms=None):
    """The record of one configuration: clean and instrumented ms per layer, per-kernel
    figures, the layer's roofline fraction and its flops dense and at the valid lengths."""
    inp = wl.inp
    kernels, flops, t_ideal = kernel_record(inp, kernel_ms, peaks, wl.out_bytes, in_step_ms)
    dense = sum(flops.values())
    at_l = valid_work(inp.lengths, inp.c_z, inp.c_h)
    return {"config": workload_config(inp, "bf16 operands, fp16 a/b/x, fp32 accumulation"),
            "directions": list(wl.dirs), "ms_per_layer": layer_ms, "ms_per_layer_instrumented": instr_layer_ms,
            "effective_tflops": dense / (layer_ms * 1e-3) / 1e12,
            "flops_dense": dense, "flops_at_valid_length": at_l,
            "tflops_at_valid_length": at_l / (layer_ms * 1e-3) / 1e12,
            "layer_roofline_frac": t_ideal / (layer_ms * 1e-3), "kernels": kernels, "l2": wl.l2_note()}


def run_ours(args):
    import datetime

    import torch

    from protein_pair_representation_b200 import trimul as tm

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def sync_all():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    out_dt = torch.float32 if args.out_dtype == "f32" else torch.bfloat16
    wl = Workload(tm, args.workload, rank, dev, out_dt, args.skip_masked)   # every replica its own seeded problem
    inp, dirs = wl.inp, wl.dirs
    for s in range(args.warmup):
        wl.step(s)
    tm.check_device_status()
    smi_index = local
    if os.environ.get("CUDA_VISIBLE_DEVICES"):
        try:
            smi_index = int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
        except ValueError:
            pass
    clocks = ClockSampler(smi_index)
    clocks.start()
    time.sleep(0.4)
    # the headline: nothing but the forwards in the timed region
    elapsed, _ = time_steps(wl, args.steps, args.warmup, sync_all, dist, dev)
    clock_info = clocks.stop()
    tm.check_device_status()
    # the per-kernel breakdown: the same steps with events between the kernels
    instr_elapsed, in_step_ms = time_steps(wl, args.steps, args.warmup + args.steps, sync_all, dist, dev,
                                           instrumented=True)
    tm.check_device_status()
    # each kernel alone, back to back through its stage entry point
    kernel_ms = stage_times(tm, wl, args.steps, sync_all)
    tm.check_device_status()
    vl = None if args.skip_masked else valid_length_pass(tm, wl, args.steps, sync_all)
    tm.check_device_status()
    out_bf16 = bf16_out_pass(tm, wl, args.steps, sync_all, measured_peaks()) if args.out_dtype == "f32" else None
    tm.check_device_status()
    warm = warm_l2_pass(wl, args.steps, sync_all)
    tm.check_device_status()

    # host-buffer end to end: every step copies its inputs in from pinned host memory and both
    # results back. A caller streams those copies: step s + 1's inputs go up and step s - 1's
    # results come down on their own streams while step s computes (two device buffer sets,
    # ordered by events), so the PCIe transfers, not the kernels, set the pace.
    e2e = None
    if not args.no_e2e:
        z_host = wl.z0.cpu().pin_memory()
        m_host = wl.m0.cpu().pin_memory()
        out_host = [[torch.empty(wl.z0.shape, dtype=out_dt, pin_memory=True) for _ in dirs] for _ in range(2)]
        zd = [wl.zs[0], torch.empty_like(wl.z0)]
        md = [wl.ms[0], torch.empty_like(wl.m0)]
        outd = [wl.outs, [torch.empty_like(o) for o in wl.outs]]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_done, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        for e_ in in_done + cmp_done + out_done:     # recorded once so that every wait has an event
            e_.record()

        def e2e_run(nsteps):
            for s_ in range(nsteps):
                i = s_ & 1
                with torch.cuda.stream(s_in):
                    s_in.wait_event(cmp_done[i])          # step s - 2 no longer reads buffer set i
                    zd[i].copy_(z_host, non_blocking=True)
                    md[i].copy_(m_host, non_blocking=True)
                    in_done[i].record()
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(in_done[i])
                    s_cmp.wait_event(out_done[i])         # step s - 2's results have been read out
                    for di, d in enumerate(dirs):
                        wl.layer.forward(zd[i], md[i], d, out=outd[i][di], stream=s_cmp)
                    cmp_done[i].record()
                with torch.cuda.stream(s_out):
                    s_out.wait_event(cmp_done[i])
                    for di in range(len(dirs)):
                        out_host[i][di].copy_(outd[i][di], non_blocking=True)
                    out_done[i].record()
            cur = torch.cuda.current_stream()
            for e_ in out_done + cmp_done + in_done:
                cur.wait_event(e_)

        e2e_run(max(2, args.warmup))
        sync_all()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for st_ in (s_in, s_cmp, s_out):
            st_.wait_event(e0)
        e2e_run(args.steps)
        e1.record()
        sync_all()
        e_el = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        e2e = {"value": job_ms_per_layer(e_el, args.steps, len(dirs), world), "unit": "ms/layer",
               "h2d_bytes_per_step": z_host.numel() * 2 + m_host.numel() * 2,
               "d2h_bytes_per_step": sum(o.numel() * o.element_size() for o in out_host[0]),
               "how": "inputs up, results down on their own streams, overlapping the neighbouring steps"}
        del zd[1], md[1], outd[1]
        torch.cuda.empty_cache()

    pair = None if args.no_pair_update else pair_update_leg(tm, wl.layer, wl.zs, wl.ms, wl.n_sets, args, dev)
    trans = None if (args.no_transition or inp.c_z != 128) else transition_leg(tm, wl.zs, wl.ms, wl.n_sets, args, dev)
    context = None if args.no_torch_context else torch_composition_leg(wl.zs, wl.ms, wl.w, inp.eps, dirs, wl.n_sets, args)

    peaks = measured_peaks()
    workloads = None
    if world == 1 and not args.no_workloads:
        workloads = {}
        for name in EXTRA_WORKLOADS:
            if name == args.workload:
                continue
            try:
                other = Workload(tm, name, 0, dev, out_dt, args.skip_masked)
                for s in range(max(3, args.warmup)):
                    other.step(s)
                w_clocks = ClockSampler(smi_index)
                w_clocks.start()
                time.sleep(0.4)
                w_el, _ = time_steps(other, args.steps, 0, sync_all)
                w_iel, w_kms = time_steps(other, args.steps, args.steps, sync_all, instrumented=True)
                w_alone = stage_times(tm, other, args.steps, sync_all)
                w_vl = None if args.skip_masked else valid_length_pass(tm, other, args.steps, sync_all)
                w_clock_info = w_clocks.stop()
                tm.check_device_status()
                n_layers = args.steps * len(other.dirs)
                workloads[name] = workload_summary(other, w_el / n_layers, w_alone, w_iel / n_layers, peaks, w_kms)
                workloads[name]["valid_lengths"] = w_vl
                workloads[name]["clocks"] = w_clock_info
                del other
                torch.cuda.empty_cache()
            except Exception as exc:        # the headline line must not depend on this leg
                workloads[name] = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in CPU_BASELINE_WORKLOADS:
        ms_cpu, cores = cpu_oracle_layer_ms(inp, dirs)
        runs = ([(w, t) for w in ("fp32_n64",) + CPU_BASELINE_WORKLOADS for t in (0, 1)] if args.cpu_full
                else list(CPU_DEFAULT_RUNS))
        cpu = {"value": ms_cpu, "unit": "ms/layer", "cores": cores, "kind": "oracle",
               "sample": f"one full layer per direction ({', '.join(dirs)}) of the same workload, fp64, "
                         f"wall clock on {cores} threads",
               "cpu_model": cpu_model(), "nproc": os.cpu_count(),
               "per_config": cpu_oracle_runs(runs)}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    n_layers = args.steps * len(dirs)
    layer_ms = job_ms_per_layer(elapsed, args.steps, len(dirs), world)
    layer_ms_single = elapsed / n_layers
    kernels, flops, t_ideal = kernel_record(inp, kernel_ms, peaks, wl.out_bytes, in_step_ms)
    nbytes = {k: kernels[k]["bytes"] for k in KERNEL_NAMES}
    dom = max(KERNEL_NAMES, key=lambda k: kernel_ms[k])
    kd = kernels[dom]
    if kd["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": kd["GB_s"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": kd["hbm_frac"], "peak_source": f"{peaks['source']} (HBM copy)"}
    else:
        roof = {"kernel": dom, "bound": "tensor", "achieved": kd["TFLOP_s"], "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": kd["tensor_frac"], "peak_source": f"{peaks['source']} (bf16 burst; fp16 equal)"}
    roof["traffic"] = recorded_traffic(dom)
    roof["algorithmic_bytes"] = nbytes[dom]
    roof["timing"] = ("mean duration of the kernel launched alone, back to back through its stage entry point, "
                      f"over {args.steps} launches between CUDA events on its stream, inputs cycling beyond the L2; "
                      "in_step_ms in `kernels` is the same kernel between events inside the forwards, where the "
                      "events also stop the next launch from overlapping its prologue")
    dense = sum(flops.values())
    at_l = valid_work(inp.lengths, inp.c_z, inp.c_h)
    cfg = workload_config(inp, "bf16 operands, fp16 a/b/x, fp32 accumulation")
    cfg.update({"out_dtype": args.out_dtype, "parallelism": f"replicas x{world}", "mask_skipping": args.skip_masked,
                "l2": wl.l2_note()})
    launches_per_forward = tm.kernels_per_forward() + (1 if args.skip_masked else 0)
    line = {
        "metric": METRIC, "value": layer_ms, "unit": "ms/layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "effective_tflops": dense / (layer_ms_single * 1e-3) / 1e12 * world,
        "flops_dense": dense, "flops_at_valid_length": at_l,
        "tflops_at_valid_length": at_l / (layer_ms_single * 1e-3) / 1e12 * world,
        "layer_roofline_frac": t_ideal / (layer_ms_single * 1e-3),
        "ms_per_layer_instrumented": instr_elapsed / n_layers,
        "kernels_alone_sum_ms": sum(kernel_ms.values()),
        "valid_lengths": vl,
        "out_bf16": out_bf16,
        "warm_l2": warm,
        "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e, "pair_update": pair,
        "pair_transition": trans, "torch_composition": context, "workloads": workloads,
        "gpu_launches": args.steps * len(dirs) * launches_per_forward,
        "clocks": clock_info,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.cpu_oracle_probe:
        cpu_oracle_probe(*args.cpu_oracle_probe)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
