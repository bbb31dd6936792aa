"""Benchmark of the triangle multiplicative update on B200 (one JSON line on rank 0).

A step is one pass of the hot path over one batch of synthetic input: the outgoing and
the incoming update (tri_mul_forward twice, three kernels each) on the OpenFold-shaped
pair workload B=1, N=512, c_z=c_h=128, bf16 z with a ragged padding mask. `value` is
milliseconds per layer (one direction) for the whole job; several GPUs run independent
replicas (weak scaling, no collective on the data path).

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
    return ap.parse_args()


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
        "cpu_baseline": {"value": ms_layer, "unit": "ms/layer", "cores": cores, "kind": "oracle", "sample": sample},
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
        nbytes = P * (2 * 128 + 2 + 2 * 128)           # z in, mask, out (bf16)
        flops = P * 2 * 2 * 128 * 256
        peaks = measured_peaks()
        gbs, tfs = nbytes / (ms * 1e-3) / 1e9, flops / (ms * 1e-3) / 1e12
        pt.close()
        return {"ms": ms, "GB_s": gbs, "TFLOP_s": tfs, "hbm_frac": gbs / peaks["hbm_gbs"],
                "tensor_frac": tfs / peaks["bf16_tflops"], "bytes": nbytes, "flops": flops,
                "traffic": recorded_traffic("pair_transition_kernel"),
                "shape": "c=128, hidden=256, bf16 in/out, fp16 hidden activation on chip"}
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


def run_ours(args):
    import datetime

    import numpy as np
    import torch

    import trimul_inputs as ti
    from protein_pair_representation_b200 import trimul as tm

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    inp = ti.make_config(args.workload, seed=rank)     # every replica its own seeded problem
    dirs = ti.CONFIGS[args.workload]["directions"]
    out_dt = torch.float32 if args.out_dtype == "f32" else torch.bfloat16
    z0 = torch.from_numpy(inp.z).to(dev).to(torch.bfloat16)
    m0 = torch.from_numpy(inp.mask).to(dev).to(torch.bfloat16)
    w = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev).to(torch.bfloat16) for k, v in inp.weights.items()}
    layer = tm.TriMulLayer(w, eps=inp.eps)
    layer.ensure_workspace(inp.B, inp.N, torch.bfloat16)
    if args.skip_masked:
        layer.set_mask_skipping(True)
    # inputs cycle through enough copies that every step reads z from outside L2
    set_bytes = z0.numel() * 2 + m0.numel() * 2
    n_sets = max(2, -(-2 * L2_BYTES // set_bytes))
    zs = [z0] + [z0.clone() for _ in range(n_sets - 1)]
    ms_ = [m0] + [m0.clone() for _ in range(n_sets - 1)]
    outs = [torch.empty(z0.shape, dtype=out_dt, device=dev) for _ in dirs]

    def step(s, evs=None):
        for di, d in enumerate(dirs):
            if evs is not None:
                layer.set_timing_events(evs[di])
            layer.forward(zs[s % n_sets], ms_[s % n_sets], d, out=outs[di])
        if evs is not None:
            layer.set_timing_events(None)

    def sync_all():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for s in range(args.warmup):
        step(s)
    tm.check_device_status()
    kev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in dirs] for _ in range(args.steps)]
    for ev in kev:                       # torch creates the CUDA event on first record
        for row in ev:
            for e in row:
                e.record()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    smi_index = local
    if os.environ.get("CUDA_VISIBLE_DEVICES"):
        try:
            smi_index = int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
        except ValueError:
            pass
    clocks = ClockSampler(smi_index)
    clocks.start()
    time.sleep(0.4)
    sync_all()
    t0.record()
    for s in range(args.steps):
        step(args.warmup + s, kev[s])
    t1.record()
    sync_all()
    clock_info = clocks.stop()
    tm.check_device_status()
    elapsed = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    kernel_ms = {k: statistics.mean(ev[d][i].elapsed_time(ev[d][i + 1]) for ev in kev for d in range(len(dirs)))
                 for i, k in enumerate(KERNEL_NAMES)}

    # host-buffer end to end: pinned inputs in, results out, every step
    e2e = None
    if not args.no_e2e:
        z_host = z0.cpu().pin_memory()
        m_host = m0.cpu().pin_memory()
        out_host = [torch.empty(z0.shape, dtype=out_dt, pin_memory=True) for _ in dirs]

        def e2e_step():
            zs[0].copy_(z_host, non_blocking=True)
            ms_[0].copy_(m_host, non_blocking=True)
            for di, d in enumerate(dirs):
                layer.forward(zs[0], ms_[0], d, out=outs[di])
                out_host[di].copy_(outs[di], non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        sync_all()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            e2e_step()
        e1.record()
        sync_all()
        e_el = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        e2e = {"value": job_ms_per_layer(e_el, args.steps, len(dirs), world), "unit": "ms/layer",
               "h2d_bytes_per_step": z_host.numel() * 2 + m_host.numel() * 2,
               "d2h_bytes_per_step": sum(o.numel() * o.element_size() for o in out_host)}

    pair = None if args.no_pair_update else pair_update_leg(tm, layer, zs, ms_, n_sets, args, dev)
    trans = None if (args.no_transition or inp.c_z != 128) else transition_leg(tm, zs, ms_, n_sets, args, dev)
    context = None if args.no_torch_context else torch_composition_leg(zs, ms_, w, inp.eps, dirs, n_sets, args)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in CPU_BASELINE_WORKLOADS:
        ms_cpu, cores = cpu_oracle_layer_ms(inp, dirs)
        cpu = {"value": ms_cpu, "unit": "ms/layer", "cores": cores, "kind": "oracle",
               "sample": f"one full layer per direction ({', '.join(dirs)}) of the same workload, fp64, "
                         f"wall clock on {cores} threads"}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = measured_peaks()
    out_bytes = 4 if out_dt == torch.float32 else 2
    flops, nbytes = layer_work(inp.B, inp.N, inp.c_z, inp.c_h, out_bytes)
    layer_ms = job_ms_per_layer(elapsed, args.steps, len(dirs), world)
    layer_ms_single = elapsed / (args.steps * len(dirs))
    kernels = {}
    for k in KERNEL_NAMES:
        t = kernel_ms[k] * 1e-3
        t_hbm = nbytes[k] / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops[k] / (peaks["bf16_tflops"] * 1e12)
        kernels[k] = {"ms": kernel_ms[k], "GB_s": nbytes[k] / t / 1e9, "TFLOP_s": flops[k] / t / 1e12,
                      "hbm_frac": nbytes[k] / t / 1e9 / peaks["hbm_gbs"],
                      "tensor_frac": flops[k] / t / 1e12 / peaks["bf16_tflops"],
                      "bound": "hbm" if t_hbm >= t_tc else "tensor", "roofline_frac": max(t_hbm, t_tc) / t}
    dom = max(KERNEL_NAMES, key=lambda k: kernel_ms[k])
    kd = kernels[dom]
    if kd["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": kd["GB_s"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": kd["hbm_frac"], "peak_source": f"{peaks['source']} (HBM copy)"}
    else:
        roof = {"kernel": dom, "bound": "tensor", "achieved": kd["TFLOP_s"], "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": kd["tensor_frac"], "peak_source": f"{peaks['source']} (bf16 burst; fp16 equal)"}
    tr = recorded_traffic(dom)
    roof["traffic"] = tr
    roof["algorithmic_bytes"] = nbytes[dom]
    t_ideal = sum(max(nbytes[k] / (peaks["hbm_gbs"] * 1e9), flops[k] / (peaks["bf16_tflops"] * 1e12))
                  for k in KERNEL_NAMES)
    cfg = workload_config(inp, "bf16 operands, fp16 a/b/x, fp32 accumulation")
    cfg.update({"out_dtype": args.out_dtype, "parallelism": f"replicas x{world}", "mask_skipping": args.skip_masked,
                "l2": f"z and mask cycle through {n_sets} copies ({n_sets * set_bytes / 2**20:.0f} MiB > 126 MiB L2)"})
    line = {
        "metric": METRIC, "value": layer_ms, "unit": "ms/layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "effective_tflops": sum(flops.values()) / (layer_ms_single * 1e-3) / 1e12 * world,
        "layer_roofline_frac": t_ideal / (layer_ms_single * 1e-3),
        "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e, "pair_update": pair,
        "pair_transition": trans, "torch_composition": context,
        "gpu_launches": args.steps * len(dirs) * (tm.kernels_per_forward() + (1 if args.skip_masked else 0)),
        "clocks": clock_info,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
