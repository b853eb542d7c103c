"""Benchmark of one MuonClip step on B200: the Muon update of the 7B-shaped
parameter set (224 hidden matrices, 7.78e9 parameters, d_model 4096, 32
layers) plus S_max and QK-Clip of one causal MHA layer (B 4, S 4096, H 32,
dh 128), all through the C ABI.  Prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 oracle on the host cores instead (a bounded
sample of the same workload: one 4096 x 4096 matrix of the 7B-shaped set per
step).  Multi-GPU (torchrun): every rank updates its own 7B-shaped parameter
set (weak scaling, no collective on the data path); the time is the max over
ranks.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon step ms & NS TFLOP/s (% bf16 peak); elementwise GB/s; QK-max tokens/s"
WORKLOAD = ("7B-shaped Muon step (224 matrices, 7.78e9 params, bf16 W/G, fp32 M, 5 NS iterations) "
            "+ causal MHA S_max and QK-Clip (B4 S4096 H32 dh128)")


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of a
# kernel kind over ONE layer of the 7B-shaped set, from the ncu capture in
# profiles/ns_gemm_1layer_full.md (third NS iteration).  A launch at full size
# covers several layers (the engine runs the list in pieces), and traffic is
# proportional to the matrices processed, so the per-launch figure is this
# times the layers one launch covers.  Kinds without a capture of the kernel
# as it stands are absent (reported as null).
KERNEL_TRAFFIC_PER_LAYER = {"ns_gram": 1.103e9, "ns_apply": 1.700e9}

# Pieces the end-to-end step splits the gradient upload into.
E2E_CHUNKS = 16


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--layers", type=int, default=32, help="layers of the 7B-shaped set (32 = full size)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the separately timed MLA QK-Clip layer and coefficient-table step")
    return p.parse_args(argv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.file.read())) if len(r) >= 9]
        self.file.close()
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "persistence_mode": self.persistence()}

    def persistence(self):
        """The GPU's persistence mode, read (never set)."""
        try:
            out = subprocess.run(["nvidia-smi", f"--id={self.gpu}", "--query-gpu=persistence_mode",
                                  "--format=csv,noheader"], capture_output=True, text=True, timeout=10)
            return out.stdout.strip() or None
        except (OSError, subprocess.TimeoutExpired):
            return None


# --------------------------------------------------------------- workload
def ns_dense_flops(shapes, steps=5):
    f = 0.0
    for (r, c) in shapes:
        m, n = min(r, c), max(r, c)
        f += steps * (4.0 * m * m * n + 2.0 * m ** 3)
    return f


def qk_flops(B, S, D, H, dh):
    return 2.0 * 2.0 * B * S * H * dh * D + 2.0 * dh * B * H * S * (S + 1) / 2.0


def flat_views(shapes, dtype, device, fill):
    """One flat device buffer with a view per matrix (so a step's input can
    travel host->device in one copy)."""
    import torch
    total = sum(r * c for r, c in shapes)
    flat = torch.empty(total, dtype=dtype, device=device)
    fill(flat)
    views, off = [], 0
    for (r, c) in shapes:
        views.append(flat[off:off + r * c].view(r, c))
        off += r * c
    return flat, views


def make_muon_inputs(device, layers, seed):
    import torch
    from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
    shapes = wl.cfg2_shapes(layers=layers)
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 + seed)
    Wf, Ws = flat_views(shapes, torch.bfloat16, device, lambda t: None)
    for W in Ws:
        W.copy_(torch.randn(W.shape, device=device, generator=gen) * 0.02)
    # gradient: N(0, 1e-3) with a log-normal scale per stored row
    Gf, Gs = flat_views(shapes, torch.bfloat16, device, lambda t: None)
    for G in Gs:
        z = torch.randn((G.shape[0], 1), device=device, generator=gen)
        G.copy_(torch.randn(G.shape, device=device, generator=gen) * 1e-3 * torch.exp(z))
    Mf, Ms = flat_views(shapes, torch.float32, device, lambda t: t.zero_())
    return shapes, (Wf, Ws), (Gf, Gs), (Mf, Ms)


# ---------------------------------------------------------------- oracle
# One matrix of each shape class of the 7B-shaped set (index in cfg2_shapes, count in the set).
ORACLE_SAMPLE = ((0, 128), (4, 64), (6, 32))   # 4096 x 4096, 14336 x 4096 (tall), 4096 x 14336 (wide)


def oracle_sample_seconds(repeats=1, rotate=False):
    """Time the fp64 oracle on the 7B-shaped set's shape classes.  Each repeat
    runs one matrix of every class (about 20 s of CPU work), or, with
    ``rotate``, one matrix of class (repeat mod 3) only.  Returns (seconds per
    repeat, FLOPs per repeat, extrapolated seconds for the whole set from the
    last time of each class)."""
    import oracle
    from matrix_orthogonalising_optimizer_step_b200 import workloads as wl
    hp = dict(wl.HPARAMS)
    shapes = wl.cfg2_shapes()
    mats = [(i, count, [t.double().numpy() for t in wl.cfg2_matrix(i)]) for i, count in ORACLE_SAMPLE]
    ts, fl, last = [], [], {}
    for r in range(repeats):
        picked = [mats[r % len(mats)]] if rotate else mats
        total = 0.0
        for i, count, (W, G, M) in picked:
            t0 = time.perf_counter()
            oracle.muon_step(W, G, M, **hp)
            dt = time.perf_counter() - t0
            total += dt
            last[i] = (dt, count)
        ts.append(total)
        fl.append(ns_dense_flops([shapes[i] for i, _, _ in picked]))
    full = sum(dt * count for dt, count in last.values()) if len(last) == len(mats) else None
    return ts, fl, full


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [d.get("num_threads") for d in info if d.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample_seconds(1, rotate=True)
    ts, fl, full = oracle_sample_seconds(args.steps, rotate=True)
    mean_s = sum(ts) / len(ts)
    value = sum(fl) / sum(ts) / 1e12
    sample = ("per step one matrix of the 7B-shaped set, the shape classes 4096x4096, 14336x4096 and "
              "4096x14336 in turn (fp64 oracle, full Muon step, 5 NS iterations)")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_s * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "sample": sample},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                            "sample": sample, "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                            "extrapolated_full_set_s": full},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# --------------------------------------------------------------- our arm
def time_extras(mc, wl, dev, stream, hp, steps, peaks, barrier, max_over_ranks, muon_set=None):
    """Work outside the step, timed on its own after the step's timed region:
    (1) S_max and the slice-map QK-Clip of a multi-head latent attention layer
    (B 4, S 4096, D 4096, H 32, content 128 + rotary 64 per head); (2) the
    64 x 1024^2 batched Muon step with its five NS coefficient triples passed
    as a per-iteration table, beside the same step with scalar coefficients;
    (3) a NorMuon step over the whole 7B-shaped set (``muon_set``: its W, G,
    M lists), whose row pass adds two bandwidth-bound kernels."""
    import torch

    out = {}
    c = wl.MLA
    B, S, D, H, dc, dr = c["B"], c["S"], c["D"], c["H"], c["dc"], c["dr"]
    X, w = wl.mla_layer_inputs()
    x = X.to(dev)
    d = {k: v.to(dev) for k, v in w.items()}
    smax = torch.empty(H, dtype=torch.float32, device=dev)
    gamma = torch.empty(H, dtype=torch.float32, device=dev)
    mask = torch.empty(H, dtype=torch.int32, device=dev)
    slices = mc.mla_slices(d["W_qC"], d["W_kC"], d["W_qR"], H, dc, dr)

    def mla_step():
        mc.mla_max_logit(x, d["W_qC"], d["W_kC"], d["W_qR"], d["W_kR"], H, dc, dr, causal=True, smax_out=smax,
                         stream=stream)
        mc.qk_clip_slices(slices, smax, H, tau=wl.QK_TAU, gamma_out=gamma, mask_out=mask, stream=stream)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        barrier()
        torch.cuda.synchronize()
        mc.profile_begin()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        k = mc.profile_end()
        assert mc.device_status() == mc.MC_OK, mc.last_error()
        barrier()
        return max_over_ranks(a.elapsed_time(b)) / reps, k

    reps = max(steps, 5)
    ms, k = timed(mla_step, reps)
    cm = k["mla_causal_max"]
    pr = k["mla_proj"]
    cm_tf = cm["flops"] / (cm["total_ms"] / 1e3) / 1e12
    out["mla_qk_clip"] = {
        "workload": f"MLA layer B{B} S{S} D{D} H{H} dc{dc} dr{dr}, causal, bf16; S_max then slice-map clip",
        "ms_per_layer": ms, "tokens_per_s": B * S / (ms / 1e3),
        "mla_causal_max_ms": cm["total_ms"] / reps, "mla_causal_max_tflops": cm_tf,
        "mla_causal_max_pct_bf16_peak": 100.0 * cm_tf / peaks["bf16_tflops"],
        "mla_proj_ms": pr["total_ms"] / reps,
        "mla_proj_tflops": pr["flops"] / (pr["total_ms"] / 1e3) / 1e12,
        "qk_clip_slices_ms": k["qk_clip_slices"]["total_ms"] / reps if "qk_clip_slices" in k else None,
        "launches_per_layer": sum(v["launches"] for v in k.values()) / reps}
    del x, d, X, w
    mc.release_workspaces()
    torch.cuda.empty_cache()

    mats = [wl.cfg1_matrix(i) for i in range(64)]
    Ws = [W.to(dev) for W, _, _ in mats]
    Gs = [G.to(dev) for _, G, _ in mats]
    Ms = [M.to(dev) for _, _, M in mats]
    table = [(hp["a"], hp["b"], hp["c"])] * hp["ns_steps"]
    res = {}
    for name, h in (("scalar", dict(hp)), ("table", dict(hp, coeffs=table))):
        ms, _ = timed(lambda: mc.muon_step(Ws, Gs, Ms, stream=stream, **h), reps)
        res[name] = ms
    flops = 64 * hp["ns_steps"] * (4 * 1024 ** 3 + 2 * 1024 ** 3)
    out["ns_coefficient_table"] = {
        "workload": "64 x 1024^2 bf16 Muon step, 5 NS iterations given as a per-iteration table",
        "ms_table": res["table"], "ms_scalar": res["scalar"],
        "tflops_dense_equiv_table": flops / (res["table"] / 1e3) / 1e12}
    del Ws, Gs, Ms
    mc.release_workspaces()
    torch.cuda.empty_cache()

    if muon_set is not None:
        Ws, Gs, Ms = muon_set
        Vs = [torch.zeros(w.shape[0], dtype=torch.float32, device=dev) for w in Ws]
        ms, k = timed(lambda: mc.normuon_step(Ws, Gs, Ms, Vs, beta2=0.95, eps_v=1e-8, stream=stream, **hp),
                      max(2, min(steps, 3)))
        reps = max(2, min(steps, 3))
        rows, app = k["normuon_rows"], k["normuon_apply"]
        out["normuon_7b"] = {
            "workload": "NorMuon step over the 7B-shaped set (224 matrices), beta2 0.95",
            "ms_per_step": ms,
            "normuon_rows_ms": rows["total_ms"] / reps,
            "normuon_rows_gbs": rows["bytes"] / (rows["total_ms"] / 1e3) / 1e9,
            "normuon_apply_ms": app["total_ms"] / reps,
            "normuon_apply_gbs": app["bytes"] / (app["total_ms"] / 1e3) / 1e9,
            "normuon_apply_pct_hbm": 100.0 * app["bytes"] / (app["total_ms"] / 1e3) / 1e9 / peaks["hbm_gbs"]}
        del Vs
        mc.release_workspaces()
        torch.cuda.empty_cache()
    return out


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import matrix_orthogonalising_optimizer_step_b200 as mc
    from matrix_orthogonalising_optimizer_step_b200 import build as mcbuild
    from matrix_orthogonalising_optimizer_step_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    mcbuild.build()
    mc.load_library()
    peaks = measured_peaks()
    hp = dict(wl.HPARAMS)

    # --- inputs (each rank its own 7B-shaped set: weak scaling)
    shapes, (Wf, Ws), (Gf, Gs), (Mf, Ms) = make_muon_inputs(dev, args.layers, seed=2 + 1000 * rank)
    n = len(shapes)
    norms = torch.zeros(n, dtype=torch.float32, device=dev)
    c3 = wl.CFG3
    B, S, D, H, dh = c3["B"], c3["S"], c3["D"], c3["H"], c3["dh"]
    X, Wq, Wk = wl.cfg3_inputs()
    x, wq, wk = X.to(dev), Wq.to(dev), Wk.to(dev)
    smax = torch.empty(H, dtype=torch.float32, device=dev)
    gamma = torch.empty(H, dtype=torch.float32, device=dev)
    mask = torch.empty(H, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        mc.muon_step(Ws, Gs, Ms, norms_out=norms, stream=stream, **hp)
        mc.qk_max_logit(x, wq, wk, H, dh, causal=True, smax_out=smax, stream=stream)
        mc.qk_clip(wq, wk, smax, H, dh, tau=wl.QK_TAU, alpha=wl.QK_ALPHA, gamma_out=gamma, mask_out=mask,
                   stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(max(args.warmup, 3)):
        step()
    assert mc.device_status() == mc.MC_OK, mc.last_error()

    # --- device-resident timed region
    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    mc.profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    kernels = mc.profile_end()
    barrier()
    clocks = sampler.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    ms_step = ms_total / args.steps
    assert mc.device_status() == mc.MC_OK, mc.last_error()

    ns_flops = ns_dense_flops(shapes, hp["ns_steps"])
    qkf = qk_flops(B, S, D, H, dh)
    step_flops = ns_flops + qkf
    value = world * step_flops / (ms_step / 1e3) / 1e12

    # --- per-kernel figures from the CUDA events around each launch
    K = args.steps
    ns_kinds = ("ns_gram", "ns_poly", "ns_apply_mixed", "ns_apply", "ns_apply_final")
    muon_kinds = ("momentum", "norm_finalize") + ns_kinds
    per = {k: dict(v, ms_per_launch=v["total_ms"] / max(v["launches"], 1)) for k, v in kernels.items()}
    ns_ms = sum(kernels[k]["total_ms"] for k in ns_kinds if k in kernels) / K
    muon_ms = sum(kernels[k]["total_ms"] for k in muon_kinds if k in kernels) / K
    ns_tflops = ns_flops / (ns_ms / 1e3) / 1e12 if ns_ms > 0 else None
    ns_exec = sum(kernels[k]["flops_executed"] for k in ns_kinds if k in kernels) / K
    ns_tflops_exec = ns_exec / (ns_ms / 1e3) / 1e12 if ns_ms > 0 else None
    mom = kernels.get("momentum")
    elem_gbs = mom["bytes"] / (mom["total_ms"] / 1e3) / 1e9 if mom else None
    qk_ms = sum(kernels[k]["total_ms"] for k in ("qk_proj", "qk_causal_max", "qk_keys") if k in kernels) / K
    qk_tokens = B * S / (qk_ms / 1e3) if qk_ms > 0 else None
    gpu_launches = sum(v["launches"] for v in kernels.values())

    # dominant kernel: the kernel kind with the largest device time
    dom = max(kernels.items(), key=lambda kv: kv[1]["total_ms"])[0]
    d = kernels[dom]
    if d["flops"] > 0:
        ach = d["flops"] / (d["total_ms"] / 1e3) / 1e12
        traffic = None
        per_layer = KERNEL_TRAFFIC_PER_LAYER.get(dom)
        iters = {"ns_gram": hp["ns_steps"], "ns_poly": hp["ns_steps"], "ns_apply_final": 1,
                 "ns_apply_mixed": min(2, hp["ns_steps"] - 1), "ns_apply": max(hp["ns_steps"] - 3, 0)}.get(dom)
        if per_layer and iters:
            launches_per_step = d["launches"] / K
            traffic = per_layer * args.layers * iters / launches_per_step
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops_sustained"], "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel timed inside a long step)"}
    else:
        ach = d["bytes"] / (d["total_ms"] / 1e3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": None, "peak_source": f"{peaks['source']} hbm_gbs"}

    # --- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        g_host = torch.empty(Gf.shape, dtype=Gf.dtype, pin_memory=True)
        g_host.copy_(Gf)
        x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        x_host.copy_(x)
        outs_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (norms, smax, gamma, mask)]
        h2d = g_host.numel() * g_host.element_size() + x_host.numel() * x_host.element_size()
        d2h = sum(t.numel() * t.element_size() for t in outs_host)
        g_host_views, off = [], 0
        for (r, c) in shapes:
            g_host_views.append(g_host[off:off + r * c].view(r, c))
            off += r * c

        def e2e_step():
            # the gradient upload overlaps the Muon step of the pieces already
            # on the device (mc_muon_step_host_grads); X goes up on the stream
            mc.muon_step_host_grads(Ws, Gs, g_host_views, Ms, chunks=E2E_CHUNKS, norms_out=norms,
                                    stream=stream, **hp)
            x.copy_(x_host, non_blocking=True)
            mc.qk_max_logit(x, wq, wk, H, dh, causal=True, smax_out=smax, stream=stream)
            mc.qk_clip(wq, wk, smax, H, dh, tau=wl.QK_TAU, alpha=wl.QK_ALPHA, gamma_out=gamma, mask_out=mask,
                       stream=stream)
            for dst, src in zip(outs_host, (norms, smax, gamma, mask)):
                dst.copy_(src, non_blocking=True)

        e2e_step()
        barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1)) / args.steps
        e2e = {"value": world * step_flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": f"muon_step_host_grads (gradient upload in {E2E_CHUNKS} pieces under the step), "
                      "qk_max_logit, qk_clip"}
        del g_host, x_host

    extras = None
    if not args.no_extras:
        extras = time_extras(mc, wl, dev, stream, hp, args.steps, peaks, barrier, max_over_ranks,
                             muon_set=(Ws, Gs, Ms))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ts, fl, full = oracle_sample_seconds(1)
        cpu = {"value": fl[0] / ts[0] / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": "one matrix of each shape class of the 7B-shaped set (4096x4096, 14336x4096, "
                         f"4096x14336), full fp64 Muon step (5 NS iterations), {ts[0]:.1f} s",
               "cpu_model": cpu_model(), "nproc": os.cpu_count(),
               "extrapolated_full_set_s": full}

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "layers": args.layers, "matrices_per_gpu": n,
                       "params_per_gpu": int(sum(r * c for r, c in shapes)),
                       "flops_per_step_per_gpu": step_flops, "flops_convention":
                           "dense-equivalent NS FLOPs 5*(4 m^2 n + 2 m^3) per matrix + QK projection and causal scores",
                       "l2": "inputs larger than L2 (about 140 GB touched per step)",
                       "parallelism": f"weak scaling, {world} independent rank(s)"},
            "components": {
                "muon_step_ms": muon_ms, "ns_tflops_dense_equiv": ns_tflops,
                "ns_pct_bf16_peak": (100.0 * ns_tflops / peaks["bf16_tflops_sustained"]) if ns_tflops else None,
                "ns_tflops_executed": ns_tflops_exec,
                "ns_pct_bf16_peak_executed": (100.0 * ns_tflops_exec / peaks["bf16_tflops_sustained"])
                if ns_tflops_exec else None,
                "elementwise_gbs": elem_gbs,
                "elementwise_pct_hbm": (100.0 * elem_gbs / peaks["hbm_gbs"]) if elem_gbs else None,
                "qk_max_tokens_per_s": qk_tokens},
            "kernels": per,
            "extras": extras,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": gpu_launches,
            "clocks": clocks,
            "peaks": peaks,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
