#!/usr/bin/env python
"""Benchmark of the Sherry 1.25-bit ternary path on B200.

Step = one batch-1 decode pass through a LLaMA-3.2-1B-shaped stack: 16 layers
x (q, k, v, o 2048x2048 / 512x2048, gate/up 8192x2048, down 2048x8192) =
112 GEMVs, 973,078,528 ternary weights, 152,043,520 bytes of codes (more than
the 126 MB L2, so no flush is needed between steps).  The codes are made on the
device by sherry_pack from seeded fp32 latents; the activations are one seeded
int8 vector per K.  Metric: packed-weight bytes streamed per second.

Also measured in the same run (rank 0): sherry_pack over all 973M fp32
latents, the two prefill GEMMs (int8 TOPS, L2 flushed between launches), the
per-projection GEMVs (L2 flushed), the end-to-end step with pinned host
buffers, and the CPU oracle on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sherry|reference]
For N > 1 run under torch.distributed.run: every rank runs its own replica of
the step (the path has no exchange step), value = all ranks' bytes / max time.
"""
import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W1.25A8 GEMV weight GB/s at batch 1 (LLaMA-3.2-1B decode stack)"
UNIT = "GB/s"
L2_BYTES = 126 * 2 ** 20
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of the timed GEMV
# kernel (gemv_dot_kernel<1,false,1>) on the 16-layer stack, B = 1, from an ncu
# capture of this kernel version (profiles/gemv_dot_decode_stack_b1.md):
# 153,628,928 read + 3,467,264 written (16-warp CTAs, nearest item boundaries).
NCU_TRAFFIC_BYTES = 153628928 + 3467264


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["sherry", "reference"], default="sherry")
    ap.add_argument("--layers", type=int, default=16)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the pack/GEMM/per-layer/CPU-baseline sub-measurements")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--gemm-only", action="store_true",
                    help="only run the two prefill GEMMs --steps times each (a small case for "
                         "profiling); prints their timings as JSON")
    ap.add_argument("--stack3b-only", type=int, default=0, metavar="B",
                    help="only run the 16-layer 3B stack at batch B for --steps steps (a case for "
                         "profiling); prints its timing as JSON")
    ap.add_argument("--mlp-chain-only", action="store_true",
                    help="only time the chained MLP blocks of --layers layers for --steps steps "
                         "(a small case for profiling); prints their JSON")
    return ap.parse_args()


def stack_spec(n_layers):
    return synth.decode_stack(n_layers)


def algorithmic_bytes(spec, B=1):
    codes = sum(n * k * 5 // 32 for _, _, n, k, _ in spec)
    scales = sum(4 * n for _, _, n, _, _ in spec)
    xs = sum(B * k for _, _, _, k, _ in spec)
    ys = sum(4 * B * n for _, _, n, _, _ in spec)
    return codes, codes + scales + xs + ys


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of the GPU this process uses (timestamps on the host).

    The GPU is matched by UUID (case and the "GPU-" prefix ignored) or by PCI
    domain/bus/device, whichever torch reports; a listing of a single GPU is
    taken as that GPU."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None, pci=None):
        self.uuid = self.norm_uuid(uuid) if uuid else None
        self.pci = pci
        self.samples = []
        self.seen = {}
        self.proc = None
        self.thread = None

    @staticmethod
    def norm_uuid(u):
        u = str(u).strip().lower()
        return u[4:] if u.startswith("gpu-") else u

    @staticmethod
    def parse_pci(bus_id):
        """'00000000:1B:00.0' -> (domain, bus, device)."""
        try:
            dom, bus, rest = bus_id.strip().split(":")
            return int(dom, 16), int(bus, 16), int(rest.split(".")[0], 16)
        except ValueError:
            return None

    def matches(self, uuid, bus_id):
        if self.uuid and self.norm_uuid(uuid) == self.uuid:
            return True
        return self.pci is not None and self.parse_pci(bus_id) == self.pci

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=uuid,pci.bus_id," + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            self.seen[parts[0]] = parts[1]
            self.samples.append((time.time(), parts[0], parts[1], parts[2:]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def select(self, samples):
        mine = [s for _, u, b, s in samples if self.matches(u, b)]
        if mine:
            return mine, "matched"
        if len(self.seen) == 1:
            return [s for _, _, _, s in samples], "only gpu listed"
        return [], "no match among %d gpus" % len(self.seen)

    def summary(self, t0, t1):
        sel, how = self.select([x for x in self.samples if t0 <= x[0] <= t1])
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "gpu": how}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(s[0]) for s in sel if num(s[0]) is not None]
        smax = [num(s[1]) for s in sel if num(s[1]) is not None]
        pw = [num(s[2]) for s in sel if num(s[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in sel for i in range(4) if s[4 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(sel), "gpu": how}


def device_keys(torch, dev):
    """(uuid, (pci domain, bus, device)) of a torch CUDA device, each None if unknown."""
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    try:
        pci = (int(props.pci_domain_id), int(props.pci_bus_id), int(props.pci_device_id))
    except (AttributeError, TypeError, ValueError):
        pci = None
    return (str(uuid) if uuid is not None else None), pci


# ----------------------------------------------------------------------------- reference arm
def max_over_ranks(value, dist=None, device=None):
    """MAX of a float over the ranks of the default process group (the value
    itself on one process)."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or \
            dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, bytes_per_step, steps, t_max):
    """Whole-job GB/s: every rank streams its own replica of the step."""
    return world * bytes_per_step * steps / t_max / 1e9


def run_reference(args, rank):
    """Times the CPU oracle on a bounded sample of the same workload."""
    import oracle
    if rank != 0:
        return None
    spec = stack_spec(args.layers)
    data = []
    for _, name, n, k, seed in spec:
        codes, scales = oracle.pack(synth.latent_weights(n, k, seed=seed))
        data.append((codes, scales, k))
    xs = {2048: synth.int8_uniform((1, 2048), seed=1), 8192: synth.int8_uniform((1, 8192), seed=2)}
    sample_bytes = sum(c.nbytes for c, _, _ in data)

    def step():
        for codes, scales, k in data:
            oracle.gemv(codes, scales, xs[k], k)
    # one step = the whole stack.  The first warm-up step sizes the run: the
    # warm-up and the timed steps asked for are each bounded to about a minute
    # of oracle time, and the line reports the counts that ran.
    t0 = time.perf_counter()
    step()
    first = time.perf_counter() - t0
    per_minute = max(1, int(60.0 / max(first, 1e-3)))
    warmup = max(1, min(args.warmup, per_minute))
    for _ in range(warmup - 1):
        step()
    steps = max(1, min(args.steps, per_minute))
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t0) / steps
    value = sample_bytes / dt / 1e9
    cores = oracle.num_threads()
    sample = "the whole stack per step (%d GEMVs, %d weights, %d code bytes), %d steps" % (
        len(spec), sum(n * k for _, _, n, k, _ in spec), sample_bytes, steps)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": "llama-3.2-1b decode stack, batch 1 (CPU oracle)", "batch": 1},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- sherry arm
def build_stack(spec, dev, S, torch, keep_latents=False):
    """Pack every layer on the device from seeded latents; return device tensors."""
    layers, latents = [], []
    for layer, name, n, k, seed in spec:
        w = torch.from_numpy(synth.latent_weights(n, k, seed=seed)).to(dev)
        codes, scales = S.pack(w)
        layers.append((layer, name, n, k, codes, scales))
        if keep_latents:
            latents.append(w)
        else:
            del w
    torch.cuda.synchronize(dev)
    return layers, latents


def time_pack(latents, layers, S, torch, peak_gbs, reps=3):
    """Packing every latent matrix of the stack (3.9 GB fp32 read): one
    sherry_pack_grouped launch (the model-load path), and one sherry_pack call
    per matrix for comparison."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    outs = [(torch.empty_like(l[4]), torch.empty_like(l[5])) for l in layers]
    grouped = S.GroupedPack([(w, c, s) for w, (c, s) in zip(latents, outs)])

    def per_matrix():
        for w, (c, s) in zip(latents, outs):
            S.pack(w, c, s)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            start.record()
            fn()
            end.record()
            end.synchronize()
            times.append(start.elapsed_time(end) / 1e3)
        return min(times)
    t = timed(grouped)
    t1 = timed(per_matrix)
    n_w = sum(l.numel() for l in latents)
    read = 4 * n_w
    written = sum(o[0].numel() * 4 + o[1].numel() * 4 for o in outs)
    return {"weights": n_w, "ms": t * 1e3, "gweights_per_s": n_w / t / 1e9,
            "gbs": (read + written) / t / 1e9, "launches": 1, "call": "sherry_pack_grouped",
            "frac_of_hbm_peak": (read + written) / t / 1e9 / peak_gbs,
            "per_matrix_calls": {"launches": len(latents), "ms": t1 * 1e3,
                                 "gbs": (read + written) / t1 / 1e9},
            "bytes_read": read, "bytes_written": written}


def l2_flusher(torch, dev):
    buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        buf.add_(1.0)
    return flush


def time_gemm(S, torch, dev, flush, reps=5):
    out = {}
    for name, M, N, K in synth.PREFILL_GEMMS:
        w = torch.from_numpy(synth.latent_weights(N, K, seed=0)).to(dev)
        codes, scales = S.pack(w)
        del w
        x = torch.from_numpy(synth.int8_clipped_normal((M, K), seed=1)).to(dev)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        for _ in range(3):
            S.gemm(codes, scales, x, y)
        torch.cuda.synchronize()
        ts = []
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(reps):
            flush()
            e0.record()
            S.gemm(codes, scales, x, y)
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) / 1e3)
        t = statistics.median(ts)
        ops = 2.0 * M * N * K
        out[name] = {"M": M, "N": N, "K": K, "ms": t * 1e3, "tops": ops / t / 1e12,
                     "bytes": M * K + N * K * 5 // 32 + 4 * N + 4 * M * N}
    return out


HBM_SPEC_GBS = 8000.0  # the B200 HBM3e figure the workload description names (~8 TB/s)


def probe_int8_tops(S, torch, iters=20000, reps=3):
    """Measured int8 tensor-core rate: sherry_probe_mma_i8 (one CTA per SM
    issuing back-to-back tcgen05 kind::i8 MMAs of the GEMM's 128 x 256 x 32
    shape, operands in shared memory), best of `reps`, in TOPS (2 ops/MAC)."""
    S.probe_mma_i8(100)
    torch.cuda.synchronize()
    best = None
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ctas = S.probe_mma_i8(iters)
        e1.record()
        e1.synchronize()
        t = e0.elapsed_time(e1) / 1e3
        best = t if best is None else min(best, t)
    macs = ctas * iters * 4 * 128 * 256 * 32
    return {"tops": 2.0 * macs / best / 1e12, "ctas": ctas, "iters": iters, "ms": best * 1e3,
            "how": "sherry_probe_mma_i8: %d CTAs x %d x 4 tcgen05.mma kind::i8 M=128 N=256 K=32, "
                   "A and B in shared memory, back to back; best of %d" % (ctas, iters, reps)}


def read_stream_gbs(torch, dev, reps=10):
    """Read-only HBM bandwidth: a 4 GiB fp32 sum, best of `reps`."""
    buf = torch.ones(1 << 30, dtype=torch.float32, device=dev)
    out = torch.empty((), dtype=torch.float32, device=dev)
    for _ in range(2):
        torch.sum(buf, dim=0, out=out)
    best = None
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.sum(buf, dim=0, out=out)
        e1.record()
        e1.synchronize()
        t = e0.elapsed_time(e1) / 1e3
        best = t if best is None else min(best, t)
    del buf
    return 4 * (1 << 30) / best / 1e9


def graph_time(torch, calls, reps):
    """Seconds per replay of a CUDA graph holding calls() (warmed up first),
    timed with events around `reps` replays."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        calls()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / 1e3 / reps


def replicas_for(nbytes):
    """Copies of a weight set that together exceed twice the L2, so that each
    call of a rotation reads its codes from HBM."""
    return max(2, -(-2 * L2_BYTES // nbytes))


def time_layers(layers, xs, S, torch, dev, reps=20):
    """Single-projection sherry_gemv calls of layer 0, B = 1: each projection
    is called on rotated copies of its codes (> 2x L2 in all) inside one CUDA
    graph, so every call reads cold codes and launch cost is the GPU's only."""
    res = {}
    for layer, name, n, k, codes, scales in layers:
        if layer != 0:
            continue
        x = xs[k]
        y = torch.empty((1, n), dtype=torch.float32, device=dev)
        ws = S.workspace(S.gemv_workspace_bytes(n, k, 1), dev)
        R = replicas_for(codes.numel() * 4)
        reps_codes = [codes.clone() for _ in range(R)]

        def calls():
            for c in reps_codes:
                S.gemv(c, scales, x, y, ws)
        t = graph_time(torch, calls, reps) / R
        del reps_codes
        cb = n * k * 5 // 32
        res[name] = {"N": n, "K": k, "us": t * 1e6, "weight_gbs": cb / t / 1e9, "copies": R}
    return res


def time_stack_single_calls(layers, xs, ys, S, torch, dev, reps=50):
    """The stack as 112 separate sherry_gemv calls (one per projection, one
    shared workspace), captured in one CUDA graph: time per step."""
    ws = S.workspace(max(S.gemv_workspace_bytes(n, k, 1) for _, _, n, k, _, _ in layers), dev)

    def calls():
        for (_, _, n, k, codes, scales), y in zip(layers, ys):
            S.gemv(codes, scales, xs[k], y, ws)
    t = graph_time(torch, calls, reps)
    code_bytes = sum(codes.numel() * 4 for _, _, _, _, codes, _ in layers)
    return {"us_per_step": t * 1e6, "weight_gbs": code_bytes / t / 1e9, "calls": len(layers),
            "steps": reps}


def time_3b_layer(S, torch, dev, reps=10):
    """One LLaMA-3.2-3B-shaped layer (7 projections, one grouped call) at
    B = 1, 4, 16 with int8 activations (seeds 1, 2, 3): rotated copies of the
    layer's codes (> 2x L2 in all), one grouped call per copy, in one CUDA
    graph."""
    items_w = []
    for pi, (name, n, k) in enumerate(synth.LLAMA_3B_LAYERS):
        w = torch.from_numpy(synth.latent_weights(n, k, seed=synth.layer_seed(0, pi))).to(dev)
        codes, scales = S.pack(w)
        del w
        items_w.append((n, k, codes, scales))
    code_bytes = sum(c.numel() * 4 for _, _, c, _ in items_w)
    R = replicas_for(code_bytes)
    copies = [[c.clone() for _, _, c, _ in items_w] for _ in range(R)]
    out = {}
    for B, seed in ((1, 1), (4, 2), (16, 3)):
        xs = {k: torch.from_numpy(synth.int8_uniform((B, k), seed=seed)).to(dev)
              for k in {k for _, k, _, _ in items_w}}
        ys = [torch.empty((B, n), dtype=torch.float32, device=dev) for n, _, _, _ in items_w]
        steps = [S.GroupedGemv([(c, s, xs[k], y) for (n, k, _, s), c, y in zip(items_w, cs, ys)], B=B)
                 for cs in copies]

        def calls():
            for st in steps:
                st()
        t = graph_time(torch, calls, reps) / R
        out["B%d" % B] = {"us": t * 1e6, "weight_gbs": code_bytes / t / 1e9}
    out["code_bytes"] = code_bytes
    out["copies"] = R
    return out


# Which activation each projection of a LLaMA layer reads: q, k and v the
# attention input, o the attention output, gate and up the MLP input, down the
# SwiGLU output.
LAYER_INPUT = {"q": "attn_in", "k": "attn_in", "v": "attn_in", "o": "attn_out",
               "gate": "mlp_in", "up": "mlp_in", "down": "mlp_act"}


def layer_activations(torch, dev, entries, B, make, seed):
    """One activation tensor per (layer, LLaMA input): the projections of a
    layer that read the same input get the same tensor, as in the model
    (q, k, v share one, gate and up another), so a grouped call prepares each
    distinct input once.  entries: (layer, projection name, K) in stack order;
    make(shape, gen) draws a tensor on the device.  Returns one tensor per entry."""
    gen = torch.Generator(device=dev).manual_seed(seed)
    made, out = {}, []
    for layer, name, k in entries:
        key = (layer, LAYER_INPUT[name])
        if key not in made:
            made[key] = make((B, k), gen)
        out.append(made[key])
    return out


def time_3b_stack(S, torch, dev, peak_gbs, n_layers=16, reps=200, batches=(1, 4, 16)):
    """A 16-layer LLaMA-3.2-3B-shaped stack (7 projections per layer, 252 MB of
    codes > L2) at B = 1, 4, 16: one grouped call per step (re-order launch +
    GEMV launch), back to back.  The codes are random words on the device
    (every word is a valid code; the kernels' work does not depend on the
    values), so no latents need to be made on the host.  Activations: int8
    uniform in [-127, 127], one per (layer, LLaMA input), shared as in the model."""
    g = torch.Generator(device=dev).manual_seed(7)
    mats = []
    for layer in range(n_layers):
        for name, n, k in synth.LLAMA_3B_LAYERS:
            codes = torch.randint(-2 ** 31, 2 ** 31 - 1, ((n + 31) // 32, k // 128, 5, 32),
                                  dtype=torch.int32, device=dev, generator=g)
            scales = torch.rand(n, device=dev, generator=g) * 0.05 + 1e-3
            mats.append((n, k, codes, scales))
    code_bytes = sum(c.numel() * 4 for _, _, c, _ in mats)
    out = {"layers": n_layers, "code_bytes": code_bytes, "codes": "random words on the device"}
    for B in batches:
        seed = {1: 1, 4: 2, 16: 3}.get(B, B)
        entries = [(l, name, k) for l in range(n_layers) for name, _, k in synth.LLAMA_3B_LAYERS]
        xs = layer_activations(torch, dev, entries, B,
                               lambda shape, gen: torch.randint(-127, 128, shape, dtype=torch.int8,
                                                                device=dev, generator=gen), seed)
        ys = [torch.empty((B, n), dtype=torch.float32, device=dev) for n, _, _, _ in mats]
        step = S.GroupedGemv([(c, s, x, y) for (n, k, c, s), x, y in zip(mats, xs, ys)], B=B)
        for _ in range(5):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            step()
        e1.record()
        e1.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / reps
        step.prepare()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            step.run()
        e1.record()
        e1.synchronize()
        tk = e0.elapsed_time(e1) / 1e3 / reps
        alg = code_bytes + sum(4 * n + B * k + 4 * B * n for n, k, _, _ in mats)
        out["B%d" % B] = {"us_per_step": t * 1e6, "weight_gbs": code_bytes / t / 1e9,
                          "kernel_us": tk * 1e6, "kernel_gbs_algorithmic": alg / tk / 1e9,
                          "frac_of_hbm": alg / tk / 1e9 / peak_gbs,
                          "kernel": "gemv_dot_kernel" if B <= 2 else "gemv_pipe_kernel"}
        del step, ys
    del mats
    torch.cuda.empty_cache()
    return out


def time_bf16_stack(layers, S, torch, dev, reps=200):
    """The same stack with bf16 activations: each step quantizes every distinct
    activation per token (fused into the re-order launch) and runs the GEMVs.
    One bf16 input per (layer, LLaMA input), shared as in the model."""
    xb = layer_activations(torch, dev, [(l, name, k) for l, name, _, k, _, _ in layers], 1,
                           lambda shape, gen: torch.randn(shape, generator=gen, device=dev).to(
                               torch.bfloat16), 3)
    ys = [torch.empty((1, n), dtype=torch.float32, device=dev) for _, _, n, _, _, _ in layers]
    items = [(codes, scales, x, y) for (_, _, n, k, codes, scales), x, y in zip(layers, xb, ys)]
    step = S.GroupedGemvBf16(items, B=1)
    for _ in range(5):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        step()
    e1.record()
    e1.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    code_bytes = sum(codes.numel() * 4 for _, _, _, _, codes, _ in layers)
    return {"us_per_step": t * 1e6, "weight_gbs": code_bytes / t / 1e9, "steps": reps,
            "note": "bf16 activations (one per layer input, seed 3) quantized per token inside the step"}


def time_mlp_chain(layers, S, torch, dev, reps=200):
    """The MLP blocks of the stack chained as a decoder runs them: per layer
    one grouped bf16 GEMV over gate and up (its kernel quantizes x), then the
    down projection on h = silu(g) * u, formed and quantized per token in its
    re-order launch (3 launches per layer; one bf16 input x for every layer)."""
    gen = torch.Generator(device="cpu").manual_seed(4)
    x = torch.randn((1, 2048), generator=gen).to(torch.bfloat16).to(dev)
    by_layer = {}
    for layer, name, n, k, codes, scales in layers:
        by_layer.setdefault(layer, {})[name] = (n, k, codes, scales)
    blocks, code_bytes = [], 0
    for layer in sorted(by_layer):
        p = by_layer[layer]
        ni = p["gate"][0]
        g = torch.empty((1, ni), dtype=torch.float32, device=dev)
        u = torch.empty((1, ni), dtype=torch.float32, device=dev)
        y = torch.empty((1, p["down"][0]), dtype=torch.float32, device=dev)
        gu = S.GroupedGemvBf16([(p["gate"][2], p["gate"][3], x, g), (p["up"][2], p["up"][3], x, u)],
                               B=1)
        dn = S.GroupedGemvF32([(p["down"][2], p["down"][3], g, u, y)], B=1)
        blocks.append((gu, dn))
        code_bytes += sum(p[m][2].numel() * 4 for m in ("gate", "up", "down"))

    def step():
        for gu, dn in blocks:
            gu()
            dn()
    for _ in range(5):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        step()
    e1.record()
    e1.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    tg = graph_time(torch, step, reps)
    return {"us_per_step": t * 1e6, "us_per_layer": t * 1e6 / len(blocks),
            "weight_gbs": code_bytes / t / 1e9, "code_bytes": code_bytes, "steps": reps,
            "graph_us_per_step": tg * 1e6, "graph_weight_gbs": code_bytes / tg / 1e9,
            "launches_per_step": 3 * len(blocks),
            "note": "x (bf16, seed 4) -> gate, up (sherry_gemv_bf16_grouped: one launch, the "
                    "GEMV quantizes x) -> down on silu(g) * u (sherry_gemv_f32_grouped: front-end "
                    "+ GEMV), layers chained"}


def time_cmp_stack(layers, xs, S, torch, dev, sherry_us, reps=500):
    """The decode stack in the two formats the pages compare Sherry against
    (2 bits per weight aligned; three weights in five bits), holding the same
    ternary matrices (transcoded on the GPU from the Sherry codes) and run by
    the same decode kernel at B = 1: one grouped call per step, back to back
    between one event pair.  The codes of each format exceed L2."""
    n_w = sum(n * k for _, _, n, k, _, _ in layers)
    sherry_bytes = sum(codes.numel() * 4 for _, _, _, _, codes, _ in layers)
    out = {"sherry": {"bits_per_weight": 8.0 * sherry_bytes / n_w, "code_bytes": sherry_bytes,
                      "us_per_step": sherry_us, "gweights_per_s": n_w / sherry_us / 1e3,
                      "weight_gbs": sherry_bytes / sherry_us / 1e3}}
    for name, fmt in (("i2_2bit", S.CMP_I2), ("t3_3in5", S.CMP_T3)):
        items, code_bytes = [], 0
        for _, _, n, k, codes, scales in layers:
            cc = S.cmp_transcode(fmt, codes, n)
            code_bytes += cc.numel() * 4
            items.append((cc, scales, xs[k], torch.empty((1, n), dtype=torch.float32, device=dev), k))
        step = S.GroupedCmpGemv(fmt, items, B=1)
        for _ in range(5):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            step()
        e1.record()
        e1.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / reps
        out[name] = {"bits_per_weight": 8.0 * code_bytes / n_w, "code_bytes": code_bytes,
                     "us_per_step": t * 1e6, "gweights_per_s": n_w / t / 1e9,
                     "weight_gbs": code_bytes / t / 1e9,
                     "sherry_speedup": t * 1e6 / sherry_us}
        del items, step
        torch.cuda.empty_cache()
    out["note"] = ("same ternary matrices in each format; one grouped decode GEMV per step "
                   "(T3 adds one activation-expansion launch, Sherry one re-order launch); "
                   "sherry_speedup = format's step time / Sherry's step time")
    return out


def _oracle_gemv_rate(host, xs_host, seconds):
    """Oracle GEMVs of the stack in stack order, repeated for ~`seconds` of
    oracle time: (GB/s of codes, GEMVs, passes started, weights, code bytes, s)."""
    import oracle
    done_bytes, done_w, n_gemv, passes, t_compute = 0, 0, 0, 0, 0.0
    while t_compute < seconds:
        for n, k, c, s in host:
            t0 = time.perf_counter()
            oracle.gemv(c, s, xs_host[k], k)
            t_compute += time.perf_counter() - t0
            done_bytes += c.nbytes
            done_w += n * k
            n_gemv += 1
            if t_compute >= seconds:
                break
        passes += 1
    return done_bytes / t_compute / 1e9, n_gemv, passes, done_w, done_bytes, t_compute


def cpu_baseline(layers, xs_host, seconds):
    """The oracle, as it stands, on bounded samples of the workloads (host
    cores).  The line's value is the decode stack on all cores; the legs add
    the stack on one thread, the pack of one layer's latents and a row slice
    of the gate/up-shaped prefill GEMM (each extrapolated to its full workload
    and labelled so)."""
    import oracle
    host = [(n, k, codes.cpu().numpy().view(np.uint32), scales.cpu().numpy())
            for _, _, n, k, codes, scales in layers]
    all_cores = oracle.num_threads()
    n_w = sum(n * k for n, k, _, _ in host)
    code_bytes = sum(c.nbytes for _, _, c, _ in host)
    v, n_gemv, passes, done_w, done_bytes, t_all = _oracle_gemv_rate(host, xs_host, 0.5 * seconds)
    legs = {"gemv_stack_all_cores": {
        "gbs": v, "cores": all_cores, "seconds": t_all,
        "stack_ms_extrapolated": code_bytes / v / 1e6,
        "sample": "%d GEMVs of the stack in stack order (%d passes started; %d weights)" % (
            n_gemv, passes, done_w)}}
    try:
        oracle.set_num_threads(1)
        v1, g1, _, w1, _, t1 = _oracle_gemv_rate(host, xs_host, 0.2 * seconds)
        legs["gemv_stack_1_thread"] = {
            "gbs": v1, "cores": 1, "seconds": t1, "stack_ms_extrapolated": code_bytes / v1 / 1e6,
            "sample": "%d GEMVs of the stack in stack order (%d weights)" % (g1, w1)}
    finally:
        oracle.set_num_threads(all_cores)
    # pack: the seven latent matrices of layer 0, best of 3
    lat = [synth.latent_weights(n, k, seed=synth.layer_seed(0, pi))
           for pi, (_, n, k) in enumerate(synth.LLAMA_1B_LAYERS)]
    best = None
    for _ in range(3):
        t0 = time.perf_counter()
        for w in lat:
            oracle.pack(w)
        t = time.perf_counter() - t0
        best = t if best is None else min(best, t)
    lw = sum(w.size for w in lat)
    legs["pack_all_cores"] = {
        "gweights_per_s": lw / best / 1e9, "gbs_read_write": (4 * lw + lw * 5 / 32) / best / 1e9,
        "cores": all_cores, "seconds": best,
        "stack_ms_extrapolated": 973078528 / (lw / best) * 1e3,
        "sample": "oracle_pack of layer 0's 7 latent matrices (%d weights), best of 3; "
                  "extrapolated to the stack's 973,078,528" % lw}
    # prefill GEMM 2048 x 8192 x 2048: a slice of 64 output rows, best of 3
    name, M, N, K = synth.PREFILL_GEMMS[0]
    rows = 64
    codes, scales = oracle.pack(synth.latent_weights(rows, K, seed=0))
    x = synth.int8_clipped_normal((M, K), seed=1)
    best = None
    for _ in range(3):
        t0 = time.perf_counter()
        oracle.gemm(codes, scales, x, K)
        t = time.perf_counter() - t0
        best = t if best is None else min(best, t)
    legs["gemm_all_cores"] = {
        "tops": 2.0 * M * rows * K / best / 1e12, "cores": all_cores, "seconds": best,
        "full_ms_extrapolated": best * (N / rows) * 1e3,
        "sample": "oracle_gemm of %d of the %d output rows of the %s GEMM (M=%d, K=%d), best of 3; "
                  "extrapolated to all rows" % (rows, N, name, M, K)}
    return {"value": v, "unit": UNIT, "cores": all_cores, "kind": "oracle", "seconds": t_all,
            "sample": legs["gemv_stack_all_cores"]["sample"] + ", %.1f s of oracle time" % t_all,
            "legs": legs}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if world > 1 and rank != 0:
            return 0
        line = run_reference(args, rank)
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from bit_gemv_sherry_b200 import sherry as S

    if args.warmup < 3:
        args.warmup = 3
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    S.lib()

    spec = stack_spec(args.layers)
    if args.gemm_only:
        flush = l2_flusher(torch, dev)
        print(json.dumps(time_gemm(S, torch, dev, flush, reps=max(1, args.steps))))
        return 0
    if args.stack3b_only:
        B = args.stack3b_only
        print(json.dumps(time_3b_stack(S, torch, dev, 6558.1, reps=max(1, args.steps),
                                       batches=(B,))))
        return 0
    if args.mlp_chain_only:
        layers, _ = build_stack(spec, dev, S, torch)
        print(json.dumps(time_mlp_chain(layers, S, torch, dev, reps=args.steps)))
        return 0
    codes_bytes, alg_bytes = algorithmic_bytes(spec)
    extras = (rank == 0) and not args.no_extras
    layers, latents = build_stack(spec, dev, S, torch, keep_latents=extras)
    xs_host = {2048: synth.int8_uniform((1, 2048), seed=1), 8192: synth.int8_uniform((1, 8192), seed=2)}
    # one device buffer for the activations and one for all outputs, so that the
    # end-to-end step moves each with a single copy
    x_all = torch.from_numpy(np.concatenate([xs_host[2048], xs_host[8192]], axis=1)).to(dev)
    xs = {2048: x_all[:, :2048], 8192: x_all[:, 2048:]}
    n_out = sum(n for _, _, n, _, _, _ in layers)
    y_all = torch.empty((n_out,), dtype=torch.float32, device=dev)
    ys, o = [], 0
    for _, _, n, _, _, _ in layers:
        ys.append(y_all[o:o + n].view(1, n))
        o += n
    items = [(codes, scales, xs[k], y) for (_, _, n, k, codes, scales), y in zip(layers, ys)]
    step = S.GroupedGemv(items, B=1)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    for _ in range(args.warmup):
        step(sptr)
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(*device_keys(torch, dev))
    clocks.start()
    time.sleep(0.3)

    K = args.steps
    # One event pair around the K timed steps, launched back to back as a decode
    # loop would run them: an event between launches would serialise the
    # programmatic dependent launch of the next kernel (the next step's re-order
    # overlaps this step's GEMV tail) and adds its own cost to every step.
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_host0 = time.time()
    e_start.record(stream)
    for i in range(K):
        step(sptr)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    t_host1 = time.time()
    if world > 1:
        dist.barrier()
    total_s = e_start.elapsed_time(e_end) / 1e3
    # The GEMV launch alone (roofline).  At B = 1 the step is that one launch
    # (the kernel re-orders each chunk's activations itself), so K2 steps back
    # to back between one event pair give its average duration (152 MB of
    # codes > L2: every launch reads HBM); for reference, the same launch
    # bracketed by its own events, and the split path (one re-order launch,
    # then GEMV launches on the prepared workspace).
    K2 = max(3, min(K, 2000))
    e_start.record(stream)
    for i in range(K2):
        step(sptr)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    gemv_s = e_start.elapsed_time(e_end) / 1e3 / K2
    K3 = max(3, min(K, 500))
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K3)]
    for i in range(K3):
        b, c = ev2[i]
        b.record(stream)
        step(sptr)
        c.record(stream)
    torch.cuda.synchronize(dev)
    gemv_bracketed_s = sum(b.elapsed_time(c) for b, c in ev2) / 1e3 / K3
    step.prepare(sptr)
    e_start.record(stream)
    for i in range(K2):
        step.run(sptr)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    run_prepared_s = e_start.elapsed_time(e_end) / 1e3 / K2
    time.sleep(0.2)
    clocks.stop()
    clk = clocks.summary(t_host0, t_host1)

    t_max = max_over_ranks(total_s, dist if world > 1 else None, dev)
    ms_per_step = t_max / K * 1e3
    value = whole_job_value(world, codes_bytes, K, t_max)

    # ---------------- end to end through the public API with pinned host buffers
    # Every step copies its activations from pinned host memory to the device,
    # runs the grouped GEMV and copies all 112 outputs back to pinned host
    # memory.  Activations and outputs alternate between two device buffers:
    # step i + 1's activations are copied in (on a copy-in stream) while step
    # i's GEMV runs, and step i's outputs are copied back (on a copy-out
    # stream) while step i + 1's GEMV runs.  A buffer is rewritten only after
    # the GEMV (activations) or the copy-back (outputs) that last read it ended.
    x_pinned = x_all.cpu().pin_memory()
    x_alt = torch.empty_like(x_all)
    xs_alt = {2048: x_alt[:, :2048], 8192: x_alt[:, 2048:]}
    y_alt = torch.empty_like(y_all)
    ys_alt, o = [], 0
    for _, _, n, _, _, _ in layers:
        ys_alt.append(y_alt[o:o + n].view(1, n))
        o += n
    step_alt = S.GroupedGemv([(codes, scales, xs_alt[k], y) for (_, _, n, k, codes, scales), y
                              in zip(layers, ys_alt)], B=1)
    e2e_steps, x_bufs, y_bufs = (step, step_alt), (x_all, x_alt), (y_all, y_alt)
    y_pinned = [torch.empty_like(y_all, device="cpu").pin_memory() for _ in range(2)]
    in_stream, out_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_ready = [torch.cuda.Event(), torch.cuda.Event()]   # activations of buffer j landed
    done = [torch.cuda.Event(), torch.cuda.Event()]      # GEMV on buffers j ended
    freed = [torch.cuda.Event(), torch.cuda.Event()]     # copy-back of outputs j ended
    h2d = x_pinned.numel()
    d2h = 4 * y_all.numel()
    K_e2e = max(3, min(K, 2000))

    def copy_in(i):
        j = i & 1
        in_stream.wait_event(done[j])          # the GEMV that last read buffer j ended
        with torch.cuda.stream(in_stream):
            x_bufs[j].copy_(x_pinned, non_blocking=True)
        x_ready[j].record(in_stream)

    def e2e_step(i, last):
        j = i & 1
        if not last:
            copy_in(i + 1)                     # next step's activations, during this GEMV
        stream.wait_event(x_ready[j])
        stream.wait_event(freed[j])            # the buffer's previous copy-back ended
        e2e_steps[j](sptr)
        done[j].record(stream)
        out_stream.wait_event(done[j])
        with torch.cuda.stream(out_stream):
            y_pinned[j].copy_(y_bufs[j], non_blocking=True)
        freed[j].record(out_stream)
    for r in range(2):
        copy_in(0)
        for i in range(4):
            e2e_step(i, i == 3)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    in_stream.wait_stream(stream)               # the first step's copy-in is inside the timed region
    copy_in(0)
    for i in range(K_e2e):
        e2e_step(i, i == K_e2e - 1)
    stream.wait_stream(out_stream)              # the last copy-back is inside the timed region
    e1.record(stream)
    e1.synchronize()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist if world > 1 else None, dev)
    if world > 1:
        dist.barrier()
    e2e_value = whole_job_value(world, codes_bytes, K_e2e, e2e_s)

    # ---------------- row-sharded step (N > 1 ranks): strong scaling of the same stack
    sharded_line = None
    if world > 1:
        from bit_gemv_sherry_b200 import sharded as SH
        parts = [SH.max_share_rows(n, world) for _, _, n, _, _, _ in layers]
        y_part = torch.zeros((sum(parts),), dtype=torch.float32, device=dev)
        y_gather = torch.empty((world * sum(parts),), dtype=torch.float32, device=dev)
        sh_items, o = [], 0
        for (_, _, n, k, codes, scales), part in zip(layers, parts):
            c_r, s_r, (n0, n1) = SH.shard(codes, scales, rank, world)
            if n1 > n0:
                sh_items.append((c_r, s_r, xs[k], y_part[o:o + n1 - n0].view(1, n1 - n0)))
            o += part
        sh_step = S.GroupedGemv(sh_items, B=1)

        def sharded_step():
            sh_step(sptr)
            dist.all_gather_into_tensor(y_gather, y_part)
        for _ in range(args.warmup):
            sharded_step()
        torch.cuda.synchronize(dev)
        dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        K_sh = max(3, min(K, 2000))
        e0.record(stream)
        for _ in range(K_sh):
            sharded_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        t_sh = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, dev)
        sharded_line = {
            "us_per_step": t_sh / K_sh * 1e6, "steps": K_sh, "scaling": "strong",
            "weight_gbs": codes_bytes * K_sh / t_sh / 1e9,
            "gather_bytes_per_rank": 4 * sum(parts),
            "note": "every projection's rows split over the %d ranks in whole 32-row groups; "
                    "per step one grouped GEMV on the shards and one NCCL all-gather of all "
                    "outputs; value = the whole stack's code bytes / max-over-ranks time" % world}
        del sh_step

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except (OSError, ValueError):
        peaks = {}
    hbm_peak = peaks.get("hbm_gbs")
    peak_src = "measured"
    if hbm_peak is None:
        hbm_peak, peak_src = 6650.0, "fallback"
    achieved = alg_bytes / gemv_s / 1e9
    # dram__bytes_read.sum + dram__bytes_write.sum of one gemv_dot_kernel launch
    # on this workload (ncu --set full); valid only for that kernel version
    ncu_traffic = NCU_TRAFFIC_BYTES if args.layers == 16 and NCU_TRAFFIC_BYTES else None

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {
            "workload": "llama-3.2-1b decode stack, batch 1: %d layers x (q,o 2048x2048; k,v "
                        "512x2048; gate,up 8192x2048; down 2048x8192)" % args.layers,
            "gemvs": len(spec), "weights": sum(n * k for _, _, n, k, _ in spec),
            "code_bytes": codes_bytes, "batch": 1,
            "l2": "inputs larger than L2: %.0f MB of codes per step > 126 MB L2, no flush" % (
                codes_bytes / 1e6),
            "launch": "sherry_gemv_grouped: one GEMV launch per step (the kernel re-orders the "
                      "activations of each chunk itself)",
            "parallelism": "replicas x%d" % world,
        },
        "gpu_launches": K,
        "clocks": clk,
        "roofline": {"bound": "hbm",
                     "kernel": "gemv_dot_kernel<1,false,1> (sherry_gemv_grouped, in-kernel re-order)",
                     "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_source": peak_src,
                     "bytes_per_launch": alg_bytes, "kernel_us": gemv_s * 1e6,
                     "kernel_launches_timed": K2,
                     "timing": "average over back-to-back launches between one event pair",
                     "kernel_us_each_bracketed_by_events": gemv_bracketed_s * 1e6,
                     "kernel_us_prepared_run": run_prepared_s * 1e6,
                     "traffic": ncu_traffic, "traffic_unit": "bytes per launch"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": K_e2e, "ms_per_step": e2e_s / K_e2e * 1e3,
                "pipelining": "per step: H2D of x, sherry_gemv_grouped, D2H of all outputs; "
                              "activations and outputs alternate between two device buffers, the "
                              "H2D of step i+1 runs during step i's GEMV (copy-in stream) and the "
                              "D2H of step i during step i+1's GEMV (copy-out stream)"},
    }
    if sharded_line is not None:
        line["sharded_step"] = sharded_line
    if extras:
        flush = l2_flusher(torch, dev)
        line["pack"] = time_pack(latents, layers, S, torch, hbm_peak)
        del latents
        torch.cuda.empty_cache()
        line["gemm"] = time_gemm(S, torch, dev, flush)
        probe = probe_int8_tops(S, torch)
        bf16x2 = 2.0 * peaks.get("bf16_tflops", 1590.0)
        gemm_rows = {}
        for name, g in line["gemm"].items():
            gemm_rows[name] = {"achieved": g["tops"], "frac": g["tops"] / probe["tops"],
                               "frac_of_2x_bf16": g["tops"] / bf16x2, "ms": g["ms"]}
        top = max(line["gemm"].values(), key=lambda g: g["ms"])
        line["gemm_roofline"] = {
            "bound": "tensor", "kernel": "gemm_kernel (sherry_gemm)", "unit": "TOPS",
            "achieved": top["tops"], "peak": probe["tops"], "frac": top["tops"] / probe["tops"],
            "peak_source": "measured tcgen05 kind::i8 probe (this run)",
            "peak_2x_measured_bf16": bf16x2, "shapes": gemm_rows, "probe": probe,
            "ops_per_launch": "2*M*N*K (dense-equivalent; 3/4 of the products are nonzero)"}
        line["gemv_layers_rotated"] = time_layers(layers, xs, S, torch, dev)
        line["gemv_bf16_stack"] = time_bf16_stack(layers, S, torch, dev)
        line["mlp_chain"] = time_mlp_chain(layers, S, torch, dev)
        line["gemv_stack_112_calls_graph"] = time_stack_single_calls(layers, xs, ys, S, torch, dev)
        rs = read_stream_gbs(torch, dev)
        line["roofline"]["other_denominators"] = {
            "read_only_stream_gbs": rs, "frac_of_read_only_stream": achieved / rs,
            "hbm_spec_gbs": HBM_SPEC_GBS, "frac_of_spec": achieved / HBM_SPEC_GBS,
            "note": "read-only stream: torch.sum over 4 GiB of fp32 (a library kernel), best of 10"}
        line["gemv_3b_layer_rotated"] = time_3b_layer(S, torch, dev)
        line["gemv_3b_stack"] = time_3b_stack(S, torch, dev, hbm_peak)
        line["formats_compared"] = time_cmp_stack(layers, xs, S, torch, dev, ms_per_step * 1e3)
        if world == 1:
            line["cpu_baseline"] = cpu_baseline(layers, xs_host, args.cpu_seconds)
    err = S.device_error()
    if err != 0:
        line["device_error"] = err
    if rank == 0:
        print(json.dumps(line))
    del step
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
