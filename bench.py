#!/usr/bin/env python
"""Decode-step benchmark of the TokenButler hot path on B200.

One step = one decode token through all layers of the workload: for every
layer, append the new key/value (+ its K_imp row), then layer 0 attends
densely and every other layer scores all cached tokens with its producer's
importance query, selects top-k + sink + window per query head and attends
over the selected tokens.  Default workload: 32 layers, G = 4, B = 4,
L = 131072 cached tokens per sequence, Llama-3.1-8B shapes (32 query / 8 KV
heads, D = 128, d' = 32), bf16 caches, keep 30 % + sink 16 + window 64.

Inputs are seeded synthetic tensors made on the device by the shared
generator; the caches (about 86 GB) are far larger than L2, so no flush is
needed between steps.  Multi-GPU: independent replicas (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-step latency (us/layer) & KV tokens scored+attended/s; HBM GB/s vs roofline"
UNIT = "KV head-tokens scored+attended/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--length", type=int, default=131072)
    ap.add_argument("--keep", type=int, default=30)
    ap.add_argument("--variant", choices=["butler", "group"], default="butler",
                    help="per-head selection (the pages' method, default) or the per-KV-group option")
    ap.add_argument("--reuse", default=None, metavar="TAU,INTERVAL,RADIUS",
                    help="amortised selection: reuse a row's cached top-k when cos >= TAU and it is at most "
                         "INTERVAL tokens old, widened by RADIUS neighbours; the step then advances the length by "
                         "one token per decode step and the importance queries drift (see --drift)")
    ap.add_argument("--kimp", choices=["f32", "bf16"], default="f32",
                    help="K_imp cache precision: fp32 (default) or the bf16 option (half the score stream)")
    ap.add_argument("--page-size", type=int, default=0,
                    help="paged K/V caches: pages of this many tokens (a power of two >= 16) placed in a shuffled "
                         "pool, addressed through a page table; 0 (default) keeps dense caches")
    ap.add_argument("--drift", type=float, default=0.05,
                    help="with --reuse: importance query of step s = q(0) + DRIFT * noise(s)")
    ap.add_argument("--shard", action="store_true",
                    help="sequence-sharded decode: every sequence's tokens split into one contiguous range per rank "
                         "(ranks in token order, the last one appending), radix histograms and partial outputs "
                         "exchanged per layer by NCCL collectives; strong scaling of the same workload")
    ap.add_argument("--trace-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-config-rows", action="store_true",
                    help="leave out the other workloads' rows (8B-shaped L=32768, prefill path, L=128K/256K sweep)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--table", action="store_true",
                    help="instead of the step benchmark, print per-kernel times (one JSON line per row) for the "
                         "8B-shaped L=32768 case, the L=4K..256K sweep of both variants and the prefill path")
    ap.add_argument("--table-iters", type=int, default=20)
    ap.add_argument("--table-only", default=None, help="regular expression on the row names to run")
    return ap.parse_args()


def workload(args):
    from query_aware_sparse_decode_b200 import synth as S
    base = S.DECODE32_B4_L128K
    wl = base.with_(n_layers=args.layers, B=args.batch, L=args.length, keep_pct=args.keep)
    if (wl.n_layers, wl.B, wl.L, wl.keep_pct) != (base.n_layers, base.B, base.L, base.keep_pct):
        wl = wl.with_(name=f"decode{wl.n_layers}_bf16_B{wl.B}_L{wl.L}_keep{wl.keep_pct}")
    if getattr(args, "variant", "butler") == "group":
        wl = wl.with_(name=wl.name + "_group_select")
    if getattr(args, "reuse", None):
        wl = wl.with_(name=wl.name + f"_reuse{args.reuse.replace(',', '_')}_drift{args.drift:g}")
    if getattr(args, "page_size", 0):
        wl = wl.with_(name=wl.name + f"_paged{args.page_size}")
    if getattr(args, "kimp", "f32") == "bf16":
        wl = wl.with_(name=wl.name + "_kimpbf16")
    return wl


def page_caches(ctx, wl, bufs, page, max_len, dev):
    """Re-bind every layer with its K/V rows moved into a pool of shuffled
    pages and a page table (K_imp and W_K stay as they are)."""
    import torch
    npg = max_len // page
    g = torch.Generator(device="cpu").manual_seed(1234)
    for layer, (k, v, kimp, w) in enumerate(bufs):
        perm = torch.randperm(wl.B * npg, generator=g)
        pools = []
        for x in (k, v):
            staged = x.view(wl.B, wl.Hkv, npg, page, wl.D).permute(0, 2, 1, 3, 4).reshape(wl.B * npg, wl.Hkv, page,
                                                                                         wl.D)
            pool = torch.empty_like(staged)
            pool[perm.to(dev)] = staged
            del staged
            pools.append(pool)
        table = perm.view(wl.B, npg).to(torch.int32).to(dev)
        lens = ctx.seq_lens(layer)
        ctx.bind_layer_paged(layer, pools[0], pools[1], table, kimp, w)
        ctx.set_seq_lens(layer, lens)
        bufs[layer] = (pools[0], pools[1], kimp, w, table)
        del k, v
    torch.cuda.empty_cache()


def variant_code(args):
    from query_aware_sparse_decode_b200 import tb as TB
    return TB.TB_BUTLER_GROUP if getattr(args, "variant", "butler") == "group" else TB.TB_BUTLER


def step_counts(wl):
    """(scored, attended) head-token pairs of one step."""
    scored = attended = 0
    k = (wl.keep_pct * wl.L) // 100
    sel = min(wl.L, wl.sink + wl.window + min(k, max(wl.L - wl.sink - wl.window, 0)))
    for layer in range(wl.n_layers):
        if layer in wl.dense_layers or wl.keep_pct == 100:
            attended += wl.B * wl.Hq * wl.L
        else:
            scored += wl.B * wl.Hq * wl.L
            attended += wl.B * wl.Hq * sel
    return scored, attended


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def begin(self, timeout: float = 2.0):
        """Waits (bounded) for the sampler's first line, then marks the start
        of the timed region: only samples from here on are summarised."""
        t_end = time.time() + timeout
        while self.proc is not None and not self.lines and time.time() < t_end:
            time.sleep(0.01)
        self.first = len(self.lines)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # a timed region shorter than the 200 ms period may see no sample: wait
        # (bounded) for the one that follows it
        first = getattr(self, "first", 0)
        t_end = time.time() + 0.5
        while len(self.lines) <= first and time.time() < t_end:
            time.sleep(0.01)
        self.lines = self.lines[first:]
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def read_peak():
    """(HBM GB/s, source): the measured copy bandwidth of MEASURED_PEAKS.json,
    else the pool's earlier measurement (fallback)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def gpu_ident(dev, local_rank: int) -> str:
    """nvidia-smi's id of the device (its UUID; the local rank otherwise)."""
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(local_rank)


# ----------------------------------------------------------------------- DRAM traffic
# DRAM bytes (read + write) per union K/V row of the sparse attention kernel,
# from one ncu capture of it (B = 2, L = 131072, keep 30 %; summary under
# profiles/).  Valid only for the kernel source it was measured on; any
# change makes it null.
ATTN_TRAFFIC = {"source_sha256_16": "8da21a82852afdd5", "bytes_per_union_row": (811.624448e6 + 3.596544e6) / 1581259}


def attn_traffic_per_row():
    import hashlib
    path = os.path.join(ROOT, "query_aware_sparse_decode_b200", "csrc", "kernels", "attn.cuh")
    with open(path, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    return ATTN_TRAFFIC["bytes_per_union_row"] if sha == ATTN_TRAFFIC["source_sha256_16"] else None


# ----------------------------------------------------------------------- ranks
def max_over_ranks_of(x: float, world: int, device) -> float:
    """Largest value of `x` over all ranks (timing is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


# ----------------------------------------------------------------------- GPU arm
def kimp_elem_bytes(cfg) -> int:
    """Bytes of one K_imp element: fp32, or bf16 with the bf16 K_imp option."""
    return 2 if cfg.kimp_bf16 else 4


def build(wl, max_len, dev, variant=None, kimp_dtype="f32"):
    import torch
    from query_aware_sparse_decode_b200 import synth as S
    from query_aware_sparse_decode_b200 import tb as TB
    cfg = TB.make_config(wl.n_layers, wl.B, wl.Hq, wl.Hkv, wl.D, wl.d_imp, wl.G, max_len, wl.dtype, wl.keep_pct,
                         wl.sink, wl.window, dense_layers=wl.dense_layers,
                         variant=TB.TB_BUTLER if variant is None else variant, kimp_dtype=kimp_dtype)
    ctx = TB.Context(cfg, dev)
    L0 = wl.L - 1
    bufs = []
    for layer in range(wl.n_layers):
        k = torch.empty((wl.B, wl.Hkv, max_len, wl.D), dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        kimp = TB.kimp_cache(cfg, dev)
        w_raw = S.w_k(wl, layer)
        w = torch.from_numpy(w_raw.view(np.int16)).view(torch.bfloat16).to(dev)
        delta = None
        if layer not in wl.dense_layers:
            # input recipe: planted keys of layer l stand out for the queries of
            # slot (l - 1) mod G of producer G * floor(l / G)
            qi = S.widen(S.q_imp(wl, wl.G * (layer // wl.G), 0), "bf16")
            qhat = qi[:, (layer - 1) % wl.G, 0, :].reshape(wl.B, wl.Hq, wl.d_imp)
            delta = torch.from_numpy(S.plant_delta(S.widen(w_raw, "bf16"), qhat, wl.Hkv)).to(dev)
        S.fill_device(k, S.K_CACHE, layer, 0, wl.B * wl.Hkv, 0, L0, wl.D, max_len * wl.D, wl.D, "bf16",
                      delta=delta, plant_mod=100 if delta is not None else 0, seed=wl.seed)
        S.fill_device(v, S.V_CACHE, layer, 0, wl.B * wl.Hkv, 0, L0, wl.D, max_len * wl.D, wl.D, "bf16",
                      seed=wl.seed)
        ctx.bind_layer(layer, k, v, kimp, w)
        ctx.set_seq_lens(layer, [L0] * wl.B)
        bufs.append((k, v, kimp, w))
    # prefill side of K_imp = K . W_K for every layer: one persistent tcgen05
    # launch over all layers, timed after one untimed launch (module load,
    # shared-memory attribute)
    ctx.project_kimp(0, 0, min(L0, 1024))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ctx.project_kimp_layers(0, wl.n_layers, 0, L0)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / wl.n_layers
    rows = wl.B * wl.Hkv * L0
    nbytes = rows * (wl.D * 2 + wl.d_imp * kimp_elem_bytes(cfg))
    proj = {"kernel": "butler_kimp_project (tcgen05, prefill of the cache, one launch over all layers)",
            "us_per_layer": us,
            "rows_per_layer": rows, "bytes_per_layer": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9,
            "tflops": 2 * rows * wl.D * wl.d_imp / (us * 1e-6) / 1e12}
    return ctx, bufs, proj


def step_inputs_host(wl, s, drift=None):
    """Pinned host tensors of step s: k_new, v_new [layers][B][Hkv][D],
    q [layers][B][Hq][D], q_imp [producers][(B*Hq)][G][1][d'].  With `drift`,
    q_imp of step s is q_imp(0) + drift * noise(s) (bf16), so consecutive
    steps' importance queries stay close."""
    import torch
    from query_aware_sparse_decode_b200 import synth as S

    def t(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
    kn, vn, qq = [], [], []
    for layer in range(wl.n_layers):
        k, v = S.kv_new(wl, layer, s)
        kn.append(k)
        vn.append(v)
        qq.append(S.query(wl, layer, s))
    nprod = (wl.n_layers + wl.G - 1) // wl.G
    if drift is None:
        qi = [S.q_imp(wl, p * wl.G, s) for p in range(nprod)]
    else:
        qi = [S.f32_to_bf16_bits((S.widen(S.q_imp(wl, p * wl.G, 0), "bf16") +
                                  drift * S.widen(S.q_imp(wl, p * wl.G, 1000 + s), "bf16")).astype(np.float32))
              for p in range(nprod)]
    return t(np.stack(kn)), t(np.stack(vn)), t(np.stack(qq)), t(np.stack(qi))


def run_step(ctx, wl, L0, inp, out, stream=None):
    """One decode step of every layer at length L0 + 1 (the new token goes to
    position L0)."""
    kn, vn, qq, qi = inp
    for layer in range(wl.n_layers):
        ctx.set_seq_lens(layer, [L0] * wl.B)
        ctx.decode_step(layer, kn[layer], vn[layer], qq[layer], qi[layer // wl.G], out[layer], stream)


def union_rows(ctx, wl, L0, inp):
    """Rows of the per-KV-head union of the selected sets (bytes attended) per
    sparse layer, measured from the library's own selection of one step."""
    import torch
    from query_aware_sparse_decode_b200 import tb as TB
    kn, vn, qq, qi = inp
    max_len = ctx.cfg.max_len
    group = ctx.cfg.variant == TB.TB_BUTLER_GROUP
    nrow = wl.Hkv if group else wl.Hq
    scores = torch.empty((wl.B, nrow, max_len), device=ctx.device)
    mask = torch.zeros((wl.B, nrow, max_len // 32), dtype=torch.int32, device=ctx.device)
    gs = wl.Hq // wl.Hkv
    rows = {}
    for layer in range(wl.n_layers):
        if layer in wl.dense_layers:
            continue
        ctx.set_seq_lens(layer, [L0 + 1] * wl.B)
        ctx.score(layer, qi[layer // wl.G], scores)
        ctx.select(layer, scores, nrow, mask=mask)
        if group:  # one set per group already
            u = mask
        else:
            m = mask.view(wl.B, wl.Hkv, gs, -1)
            u = m[:, :, 0]
            for j in range(1, gs):
                u = u | m[:, :, j]
        bits = np.unpackbits(u.cpu().numpy().view(np.uint8), bitorder="little")
        rows[layer] = int(bits.sum())
    return rows


def gpu_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from query_aware_sparse_decode_b200 import tb as TB
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workload(args)
    L0 = wl.L - 1
    max_len = (wl.L + 255) // 256 * 256
    if max_len == wl.L:
        max_len += 256
    ctx, bufs, proj = build(wl, max_len, dev, variant_code(args), args.kimp)
    if args.page_size:
        if max_len % args.page_size:
            raise SystemExit("--page-size must divide the cache capacity")
        page_caches(ctx, wl, bufs, args.page_size, max_len, dev)
    stream = torch.cuda.current_stream(dev)
    nvar = min(args.steps + args.warmup, 4)
    drift = None
    if args.reuse:  # amortised selection: caches bound, queries drifting, the length advancing
        tau, interval, radius = args.reuse.split(",")
        for layer in range(wl.n_layers):
            ctx.selection_cache(layer)
        ctx.set_reuse(float(tau), int(interval), int(radius))
        drift = args.drift
    host_inputs = [step_inputs_host(wl, s, drift) for s in range(nvar)]
    pos = {"n": 0}

    def next_L0():
        """Position of the step's new token: fixed, or advancing by one per
        step when selections are cached (max_len leaves 255 tokens of room)."""
        if not args.reuse:
            return L0
        pos["n"] += 1
        if pos["n"] >= max_len - wl.L:
            raise RuntimeError("--reuse runs out of cache room: use fewer steps")
        return L0 + pos["n"]
    dev_inputs = [tuple(x.to(dev) for x in h) for h in host_inputs]
    out = torch.empty((wl.n_layers, wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    scored, attended = step_counts(wl)
    tokens = scored + attended

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        return max_over_ranks_of(x, world, dev)

    for s in range(args.warmup):
        run_step(ctx, wl, next_L0(), dev_inputs[s % nvar], out, stream)
    barrier()

    # ---- device-timed region: inputs resident in HBM
    clocks = ClockSampler(gpu_ident(dev, local_rank))
    clocks.start()
    clocks.begin()
    n0 = ctx.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for s in range(args.steps):
        run_step(ctx, wl, next_L0(), dev_inputs[s % nvar], out, stream)
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    launches = ctx.launch_count() - n0
    ms = max_over_ranks(e0.elapsed_time(e1))
    ms_step = ms / args.steps
    value = whole_job_rate(tokens, args.steps, world, ms)

    # ---- per-kernel times (trace events inside decode_step, same workload)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(wl.n_layers)]
    seg = {"append": [], "score": [], "select": [], "attn": [], "combine": [], "attn_dense": []}
    kn, vn, qq, qi = dev_inputs[0]
    for s in range(args.trace_steps):
        Ls = next_L0()
        for layer in range(wl.n_layers):
            ctx.trace_events(ev[layer])
            ctx.set_seq_lens(layer, [Ls] * wl.B)
            ctx.decode_step(layer, kn[layer], vn[layer], qq[layer], qi[layer // wl.G], out[layer], stream)
        ctx.trace_events(None)
        torch.cuda.synchronize(dev)
        for layer in range(wl.n_layers):
            e = ev[layer]
            t = [e[i].elapsed_time(e[i + 1]) * 1e3 for i in range(5)]  # us
            seg["append"].append(t[0])
            seg["combine"].append(t[4])
            if layer in wl.dense_layers:
                seg["attn_dense"].append(t[3])
            else:
                seg["score"].append(t[1])
                seg["select"].append(t[2])
                seg["attn"].append(t[3])
    avg = {k: (sum(v) / len(v) if v else 0.0) for k, v in seg.items()}

    # ---- algorithmic bytes
    urows = union_rows(ctx, wl, L0, dev_inputs[0])
    sparse_layers = [l for l in range(wl.n_layers) if l not in wl.dense_layers]
    row_kv = 2 * wl.D * 2                                   # K + V row, bf16
    kimp_bytes = wl.B * wl.Hkv * wl.L * wl.d_imp * kimp_elem_bytes(ctx.cfg)   # per sparse layer
    union_bytes = (sum(urows.values()) / max(len(urows), 1)) * row_kv
    dense_bytes = wl.B * wl.Hkv * wl.L * row_kv
    step_bytes = len(sparse_layers) * (kimp_bytes + union_bytes) + (wl.n_layers - len(sparse_layers)) * dense_bytes
    peak, peak_src = read_peak()
    attn_gbs = union_bytes / (avg["attn"] * 1e-6) / 1e9 if avg["attn"] else None
    score_gbs = kimp_bytes / (avg["score"] * 1e-6) / 1e9 if avg["score"] else None
    pair_gbs = ((kimp_bytes + union_bytes) / ((avg["score"] + avg["attn"]) * 1e-6) / 1e9
                if avg["attn"] else None)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dbuf = tuple(torch.empty_like(x) for x in dev_inputs[0])
        h2d = sum(x.numel() * x.element_size() for x in host_inputs[0])
        d2h = out.numel() * out.element_size()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for s in range(args.steps):
            for dst, src in zip(dbuf, host_inputs[s % nvar]):
                dst.copy_(src, non_blocking=True)
            run_step(ctx, wl, next_L0(), dbuf, out, stream)
            out_host.copy_(out, non_blocking=True)
        f1.record(stream)
        barrier()
        ems = max_over_ranks(f0.elapsed_time(f1))
        e2e = {"value": whole_job_rate(tokens, args.steps, world, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems / args.steps}

    status = ctx.check_status()
    if status:
        raise RuntimeError(f"device status flags {status:#x}")
    return dict(proj=proj, wl=wl, value=value, ms_step=ms_step, clk=clk, launches=launches, avg=avg, urows=urows,
                union_bytes=union_bytes, kimp_bytes=kimp_bytes, step_bytes=step_bytes, peak=peak,
                peak_src=peak_src, attn_gbs=attn_gbs, score_gbs=score_gbs, pair_gbs=pair_gbs, e2e=e2e,
                scored=scored, attended=attended)


# ----------------------------------------------------------------------- sequence-sharded arm
def shard_arm(args, rank, world, local_rank):
    """The workload's decode step with every sequence split by token range
    over the ranks (include/tb.h, "Sequence-sharded decode"; shard.py gives
    the call order).  Rank r holds tokens [r * per, (r + 1) * per) of every
    layer's caches; per layer the ranks exchange two summed radix histograms,
    one gathered histogram and the gathered fp32 partial outputs with NCCL
    (one rank: in-process copies).  The total work is fixed: strong scaling."""
    import torch
    import torch.distributed as dist
    from query_aware_sparse_decode_b200 import synth as S
    from query_aware_sparse_decode_b200 import tb as TB
    from query_aware_sparse_decode_b200.shard import ShardBuffers, TorchCollectives, run_lockstep, shard_step
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workload(args)
    wl = wl.with_(name=wl.name + f"_sharded{world}")
    L0 = wl.L - 1
    per = (L0 + world - 1) // world
    t0 = rank * per
    n = max(0, min(per, L0 - t0))
    last = rank == world - 1
    cap = (n + 2 + 255) // 256 * 256
    cfg = TB.make_config(wl.n_layers, wl.B, wl.Hq, wl.Hkv, wl.D, wl.d_imp, wl.G, cap, wl.dtype, wl.keep_pct, wl.sink,
                         wl.window, dense_layers=wl.dense_layers)
    ctx = TB.Context(cfg, dev)
    bufs = []
    for layer in range(wl.n_layers):
        k = torch.empty((wl.B, wl.Hkv, cap, wl.D), dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        w_raw = S.w_k(wl, layer)
        delta = None
        if layer not in wl.dense_layers:
            qi = S.widen(S.q_imp(wl, wl.G * (layer // wl.G), 0), "bf16")
            qhat = qi[:, (layer - 1) % wl.G, 0, :].reshape(wl.B, wl.Hq, wl.d_imp)
            delta = torch.from_numpy(S.plant_delta(S.widen(w_raw, "bf16"), qhat, wl.Hkv)).to(dev)
        if n:
            S.fill_device(k, S.K_CACHE, layer, 0, wl.B * wl.Hkv, t0, t0 + n, wl.D, cap * wl.D, wl.D, "bf16",
                          delta=delta, plant_mod=100 if delta is not None else 0, seed=wl.seed, dst_t0=0)
            S.fill_device(v, S.V_CACHE, layer, 0, wl.B * wl.Hkv, t0, t0 + n, wl.D, cap * wl.D, wl.D, "bf16",
                          seed=wl.seed, dst_t0=0)
        kimp = TB.kimp_cache(cfg, dev)
        ctx.bind_layer(layer, k, v, kimp, torch.from_numpy(w_raw.view(np.int16)).view(torch.bfloat16).to(dev))
        ctx.set_seq_lens(layer, [n] * wl.B)
        bufs.append((k, v, kimp))
    if n:
        ctx.project_kimp_layers(0, wl.n_layers, 0, n)
    sb = ShardBuffers(cfg, world, dev)
    nvar = min(args.steps + args.warmup, 4)
    host_inputs = [step_inputs_host(wl, s) for s in range(nvar)]
    dev_inputs = [tuple(x.to(dev) for x in h) for h in host_inputs]
    out = torch.empty((wl.n_layers, wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    coll = TorchCollectives() if world > 1 else None

    def one_step(inp):
        kn, vn, qq, qi = inp
        for layer in range(wl.n_layers):
            ctx.set_seq_lens(layer, [n] * wl.B)
            st = shard_step(ctx, layer, rank, world, t0, [wl.L] * wl.B, qq[layer], qi[layer // wl.G], out[layer], sb,
                            kn[layer] if last else None, vn[layer] if last else None, stream)
            if coll is not None:
                coll.run(st)
            else:
                run_lockstep([st])

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for s in range(args.warmup):
        one_step(dev_inputs[s % nvar])
    barrier()
    clocks = ClockSampler(gpu_ident(dev, local_rank))
    clocks.start()
    clocks.begin()
    n0 = ctx.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for s in range(args.steps):
        one_step(dev_inputs[s % nvar])
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    launches = ctx.launch_count() - n0
    ms = max_over_ranks_of(e0.elapsed_time(e1), world, dev)
    scored, attended = step_counts(wl)
    value = (scored + attended) * args.steps / (ms / 1e3)   # the whole job's fixed work
    # end to end: this rank's inputs copied in from pinned memory, the merged output read back
    dbuf = tuple(torch.empty_like(x) for x in dev_inputs[0])
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for s in range(args.steps):
        for dst, src in zip(dbuf, host_inputs[s % nvar]):
            dst.copy_(src, non_blocking=True)
        one_step(dbuf)
        out_host.copy_(out, non_blocking=True)
    f1.record(stream)
    barrier()
    ems = max_over_ranks_of(f0.elapsed_time(f1), world, dev)
    status = ctx.check_status()
    if status:
        raise RuntimeError(f"device status flags {status:#x}")
    if rank == 0:
        peak, peak_src = read_peak()
        kimp_b = wl.B * wl.Hkv * wl.L * wl.d_imp * 4
        dense_b = wl.B * wl.Hkv * wl.L * 2 * wl.D * 2
        nsp = sum(1 for l in range(wl.n_layers) if l not in wl.dense_layers)
        step_bytes = nsp * kimp_b + (wl.n_layers - nsp) * dense_b
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": wl.name, "layers": wl.n_layers, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv,
                           "D": wl.D, "d_imp": wl.d_imp, "G": wl.G, "L": wl.L, "keep_pct": wl.keep_pct,
                           "sink": wl.sink, "window": wl.window, "dense_layers": list(wl.dense_layers),
                           "selection": "per_query_head, sharded by token range", "tokens_per_rank": per,
                           "parallelism": f"sequence-sharded x{world}",
                           "l2": "inputs larger than L2 (caches of all layers, no flush)"},
                "us_per_layer": ms / args.steps * 1e3 / wl.n_layers,
                "tokens_scored_per_step": scored, "tokens_attended_per_step": attended,
                "roofline": {"kernel": "a rank's whole sharded step (K_imp of sparse layers + dense K/V; the "
                                       "attended rows are not counted, a lower bound)", "bound": "hbm",
                             "achieved": step_bytes / world / (ms / args.steps * 1e-3) / 1e9, "peak": peak,
                             "unit": "GB/s", "frac": step_bytes / world / (ms / args.steps * 1e-3) / 1e9 / peak,
                             "traffic": None, "peak_source": peak_src},
                "gpu_launches": launches, "clocks": clk,
                "e2e": {"value": (scored + attended) * args.steps / (ems / 1e3), "unit": UNIT,
                        "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host_inputs[0]),
                        "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": ems / args.steps},
                "cpu_baseline": None}
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------- CPU oracle leg
def _oracle_slab(wl, layer, b, kimp):
    """Host inputs of one (layer, sequence) slab of the workload at L: the
    caches with the step's appended token, the queries and the cache's K_imp
    (projected by the oracle; a decode step finds it in the cache)."""
    from oracle import native as N
    from query_aware_sparse_decode_b200 import synth as S
    L0 = wl.L - 1
    W = S.widen(S.w_k(wl, layer), wl.dtype)
    qi = S.widen(S.q_imp(wl, N.producer_of(layer, wl.G), 0), wl.dtype)
    qhat = N.importance_queries(qi, layer, wl.G, wl.B, wl.Hq)
    delta = S.plant_delta(W, qhat, wl.Hkv)
    K = S.widen(S.kv_cache_host(wl, layer, S.K_CACHE, 0, L0, delta, b_range=(b, 1)), wl.dtype)
    V = S.widen(S.kv_cache_host(wl, layer, S.V_CACHE, 0, L0, b_range=(b, 1)), wl.dtype)
    kn, vn = S.kv_new(wl, layer, 0)
    K = np.concatenate([K, S.widen(kn, wl.dtype)[b][:, None]], axis=1)[None]
    V = np.concatenate([V, S.widen(vn, wl.dtype)[b][:, None]], axis=1)[None]
    Kimp = N.project_keys(K, W, "bf16" if kimp == "bf16" else "f64")
    q = S.widen(S.query(wl, layer, 0), wl.dtype)[b:b + 1]
    qi_b = qi.reshape(wl.B, wl.Hq, wl.G, 1, wl.d_imp)[b]
    return q, K, V, W, qi_b, Kimp


def oracle_sample(wl, seconds: float, group: bool = False, kimp: str = "f64", threads=None, max_runs: int = 64,
                  n_inputs: int = 2):
    """Times the C++ fp64 oracle (oracle/tokenbutler.cpp) on whole (layer,
    sequence) slabs of the workload: the decode step's score, select and
    attend for all query heads at L (a3-a6), with the cache's K_imp given.
    `n_inputs` slabs are generated on the host outside the timed region and
    timed in turn until about `seconds` of oracle work (at least one run,
    at most `max_runs`), with `threads` OpenMP threads (default: every core)."""
    from oracle import native as N
    nproc = os.cpu_count() or 1
    threads = nproc if threads is None else threads
    N.set_threads(nproc)  # input preparation on every core
    sparse_layers = [l for l in range(wl.n_layers) if l not in wl.dense_layers] or [0]
    inputs = []
    for i in range(n_inputs):
        layer = sparse_layers[(1 + 7 * i) % len(sparse_layers)]
        inputs.append((layer, _oracle_slab(wl, layer, i % wl.B, kimp)))
    N.set_threads(threads)
    elapsed, tokens, runs = 0.0, 0, 0
    while (elapsed < seconds or runs == 0) and runs < max_runs:
        layer, (q, K, V, W, qi_b, Kimp) = inputs[runs % n_inputs]
        t0 = time.perf_counter()
        sel, _, _, _ = N.decode_layer(q, K, V, W, qi_b, layer, wl.G, wl.L, wl.keep_pct, wl.sink, wl.window,
                                      dense=False, K_imp=Kimp, group=group)
        elapsed += time.perf_counter() - t0
        tokens += wl.Hq * wl.L + sum(len(v) for v in sel.values())
        runs += 1
    return {"value": tokens / elapsed, "unit": UNIT, "threads": threads, "runs": runs, "inputs": n_inputs,
            "seconds": elapsed}


def cpu_baseline(wl, seconds: float, group: bool = False, kimp: str = "f64"):
    """The oracle single-threaded and on every core of the host (about
    `seconds` each); the line's value is the all-core rate."""
    nproc = os.cpu_count() or 1
    single = oracle_sample(wl, seconds / 2, group, kimp, threads=1, max_runs=2, n_inputs=1)
    allc = oracle_sample(wl, seconds / 2, group, kimp, threads=nproc)
    return {"value": allc["value"], "unit": UNIT, "cores": nproc, "kind": "oracle",
            "sample": f"{allc['runs']} runs over {allc['inputs']} (layer, sequence) slabs of {wl.name} on {nproc} "
                      f"threads and {single['runs']} on one: score + select + attend (a3-a6) for all {wl.Hq} query "
                      f"heads at "
                      f"L={wl.L}, the cache's K_imp projected outside the timed region, C++ fp64 oracle, "
                      f"{allc['seconds']:.1f} s + {single['seconds']:.1f} s",
            "single": {"value": single["value"], "threads": 1},
            "all_core": {"value": allc["value"], "threads": nproc},
            "cores_nproc": nproc, "omp_num_threads": os.environ.get("OMP_NUM_THREADS")}


def reference_arm(args, rank, world):
    """The oracle as the reference arm: each step one (layer, sequence) slab
    of the workload on every host core (rank 0 only; other ranks exit)."""
    if rank != 0:
        return
    wl = workload(args)
    vals = []
    for s in range(args.warmup + args.steps):
        r = oracle_sample(wl, seconds=0.0, group=args.variant == "group", kimp=args.kimp, max_runs=1, n_inputs=1)
        if s >= args.warmup:
            vals.append(r)
    value = statistics.mean(v["value"] for v in vals)
    nproc = os.cpu_count() or 1
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "L": wl.L, "layers": wl.n_layers, "keep_pct": wl.keep_pct,
                       "sink": wl.sink, "window": wl.window},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nproc, "kind": "oracle",
                             "sample": f"each step: one (layer, sequence) slab of {wl.name}: score + select + "
                                       f"attend (a3-a6) for all {wl.Hq} query heads at L={wl.L}, the cache's K_imp "
                                       f"projected outside the timed region, C++ fp64 oracle on {nproc} threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------- per-kernel table
def _pct(xs, q):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, int(round(q * (len(xs) - 1))))]


def _timed_decode(ctx, wl, layer, inp, iters, flush_buf, stream):
    """Per-segment times (us) of single decode steps, each bracketed by the
    library's trace events; with `flush_buf`, L2 is flushed before every step
    (outside the events) by a 512 MB write followed by a 256 MB read, so the
    step starts with L2 full of clean, unrelated lines."""
    import torch
    kn, vn, qq, qi = inp
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=ctx.device)
    rows = []
    for it in range(3 + iters):
        ctx.set_seq_lens(layer, [wl.L - 1] * wl.B)
        if flush_buf is not None:
            flush_buf.add_(1)
            flush_buf.view(torch.float32)[: 64 << 20].sum()
        ctx.trace_events(ev)
        ctx.decode_step(layer, kn, vn, qq, qi, out, stream)
        ctx.trace_events(None)
        torch.cuda.synchronize()
        if it >= 3:
            rows.append([ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(5)] + [ev[0].elapsed_time(ev[5]) * 1e3])
    names = ["append", "score", "select", "attn", "combine", "total"]
    med = {n: statistics.median(r[i] for r in rows) for i, n in enumerate(names)}
    med["total_p90"] = _pct([r[5] for r in rows], 0.9)
    return med


def _cold_batched(fn, flush, reps=5, k=10):
    """Device time (us) of one call of `fn` starting with a cold L2 and no
    launch gap: `k` pairs (flush, fn) queued back to back minus `k` flushes
    queued alone, the two interleaved `reps` times, median of the
    differences.  The flush is a 256 MB read, so the call starts with L2 full
    of clean, unrelated lines; as in a chained decode step, the call's launch
    is processed while the work before it runs."""
    import torch
    e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    fn()
    flush()
    torch.cuda.synchronize()
    diffs = []
    for _ in range(reps):
        e[0].record()
        for _ in range(k):
            flush()
        e[1].record()
        for _ in range(k):
            flush()
            fn()
        e[2].record()
        torch.cuda.synchronize()
        diffs.append((e[1].elapsed_time(e[2]) - e[0].elapsed_time(e[1])) * 1e3 / k)
    return statistics.median(diffs)


def _batched_case(ctx, wl, variant, layer, inp, flush_buf, max_len):
    """Per-call cold-L2 device times (us) of the separate calls of one decode
    step (score or soft-vote logits + reduce, selection, attention + combine)
    and of the fused step, with `_cold_batched`."""
    import torch
    from query_aware_sparse_decode_b200 import tb as TB
    kn, vn, qq, qi = inp
    dev = ctx.device
    flat = flush_buf.view(torch.float32)[: 64 << 20]

    def flush():
        flat.sum()
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    gs = wl.Hq // wl.Hkv
    t = {}
    dense = wl.keep_pct >= 100 or layer in wl.dense_layers
    ctx.set_seq_lens(layer, [wl.L] * wl.B)
    if dense:
        t["attn"] = _cold_batched(lambda: ctx.sparse_attn(layer, qq, None, TB.TB_MASK_DENSE, out), flush)
    else:
        if variant == TB.TB_SOFTVOTE:
            sc = torch.empty((wl.B, max_len), device=dev)
            nrow, mode = 1, TB.TB_MASK_SHARED
            t["score"] = _cold_batched(lambda: ctx.softvote_scores(layer, qq, sc), flush)
        else:
            group = variant == TB.TB_BUTLER_GROUP
            nrow = wl.Hkv if group else wl.Hq
            mode = TB.TB_MASK_GROUP if group else TB.TB_MASK_PER_HEAD
            sc = torch.empty((wl.B, nrow, max_len), device=dev)
            t["score"] = _cold_batched(lambda: ctx.score(layer, qi, sc), flush)
        mask = torch.zeros((wl.B, nrow, max_len // 32), dtype=torch.int32, device=dev)
        t["select"] = _cold_batched(lambda: ctx.select(layer, sc, nrow, mask=mask), flush)
        t["attn"] = _cold_batched(lambda: ctx.sparse_attn(layer, qq, mask, mode, out), flush)

    def step():
        ctx.set_seq_lens(layer, [wl.L - 1] * wl.B)
        ctx.decode_step(layer, kn, vn, qq, qi, out)
    t["step"] = _cold_batched(step, flush)
    ctx.set_seq_lens(layer, [wl.L] * wl.B)
    return t


def _variant_name(variant):
    from query_aware_sparse_decode_b200 import tb as TB
    return {TB.TB_SOFTVOTE: "softvote", TB.TB_BUTLER_GROUP: "group"}.get(variant, "butler")


def _table_case(wl, variant, dev, iters, flush_buf, peak, hot_l2=True):
    import torch
    from query_aware_sparse_decode_b200 import synth as S
    from query_aware_sparse_decode_b200 import tb as TB
    max_len = (wl.L + 1 + 255) // 256 * 256
    ctx, bufs, _ = build(wl, max_len, dev, variant)
    layer = 0
    stream = torch.cuda.current_stream(dev)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    kn, vn = S.kv_new(wl, layer)
    inp = (bf(kn), bf(vn), bf(S.query(wl, layer)), bf(S.q_imp(wl, 0)))
    cold = _timed_decode(ctx, wl, layer, inp, iters, flush_buf, stream)
    hot = _timed_decode(ctx, wl, layer, inp, iters, None, stream) if hot_l2 else None
    batched = _batched_case(ctx, wl, variant, layer, inp, flush_buf, max_len)
    # algorithmic bytes from the library's own selection of this step
    ctx.set_seq_lens(layer, [wl.L] * wl.B)
    dense = wl.keep_pct >= 100 or layer in wl.dense_layers
    row_kv = 2 * wl.D * 2
    gs = wl.Hq // wl.Hkv
    if dense:
        first, union = 0, wl.B * wl.Hkv * wl.L
    elif variant == TB.TB_SOFTVOTE:
        votes = torch.empty((wl.B, max_len), device=dev)
        mask = torch.zeros((wl.B, 1, max_len // 32), dtype=torch.int32, device=dev)
        ctx.softvote_scores(layer, inp[2], votes)
        ctx.select(layer, votes, 1, mask=mask)
        first = wl.B * wl.Hkv * wl.L * wl.D * 2               # the full K, read for the logits
        union = int(np.unpackbits(mask.cpu().numpy().view(np.uint8)).sum()) * wl.Hkv
    else:
        group = variant == TB.TB_BUTLER_GROUP
        nrow = wl.Hkv if group else wl.Hq
        scores = torch.empty((wl.B, nrow, max_len), device=dev)
        mask = torch.zeros((wl.B, nrow, max_len // 32), dtype=torch.int32, device=dev)
        ctx.score(layer, inp[3], scores)
        ctx.select(layer, scores, nrow, mask=mask)
        if group:
            u = mask
        else:
            m = mask.view(wl.B, wl.Hkv, gs, -1)
            u = m[:, :, 0]
            for j in range(1, gs):
                u = u | m[:, :, j]
        first = wl.B * wl.Hkv * wl.L * wl.d_imp * kimp_elem_bytes(ctx.cfg)   # K_imp
        union = int(np.unpackbits(u.cpu().numpy().view(np.uint8)).sum())
    torch.cuda.synchronize()
    if ctx.check_status():
        raise RuntimeError("device status flags set")
    attn_bytes = union * row_kv

    def rates(t):
        r = {"attn_gbs": attn_bytes / (t["attn"] * 1e-6) / 1e9}
        if not dense:
            r["score_gbs"] = first / (t["score"] * 1e-6) / 1e9
            r["score_plus_attn_gbs"] = (first + attn_bytes) / ((t["score"] + t["attn"]) * 1e-6) / 1e9
            r["score_plus_attn_frac"] = r["score_plus_attn_gbs"] / peak
        r["attn_frac"] = r["attn_gbs"] / peak
        r["step_gbs"] = (first + attn_bytes) / (t["total"] * 1e-6) / 1e9
        return r
    bt = batched
    line = {"table": "decode", "workload": wl.name, "variant": _variant_name(variant),
            "B": wl.B, "L": wl.L, "keep_pct": wl.keep_pct, "dense": dense,
            "first_pass_bytes": first, "union_rows": union, "attn_bytes": attn_bytes,
            "us_batched": bt,
            "batched_attn_frac": attn_bytes / (bt["attn"] * 1e-6) / 1e9 / peak,
            "batched_pair_frac": (None if dense else
                                  (first + attn_bytes) / ((bt["score"] + bt["attn"]) * 1e-6) / 1e9 / peak),
            "batched_step_gbs": (first + attn_bytes) / (bt["step"] * 1e-6) / 1e9,
            "us_cold_l2": cold, "us_hot_l2": hot, "rates_cold_l2": rates(cold),
            "rates_hot_l2": rates(hot) if hot is not None else None,
            "l2": "cold: 512 MB write + 256 MB read before each step; hot: back-to-back steps",
            "iters": iters,
            "peak_gbs": peak}
    del ctx, bufs
    torch.cuda.empty_cache()
    return line


def _table_prefill(dev, iters, peak, n_layers=None):
    import torch
    from query_aware_sparse_decode_b200 import synth as S
    wl = S.PREFILL_L32K
    if n_layers is not None and n_layers < wl.n_layers:  # a smaller cache set, e.g. for a profiler
        wl = wl.with_(n_layers=max(2, n_layers))
    max_len = wl.L + 256
    # build() fills and projects rows [0, L - 1) of its workload: one more
    # gives the whole 32768-row prefix of every layer
    ctx, bufs, proj = build(wl.with_(L=wl.L + 1), max_len, dev)
    layer, nrows = 1, 1024
    row0 = wl.L - nrows
    qrows = S.q_imp(wl, 0, rows=(row0, nrows))
    qd = torch.from_numpy(np.ascontiguousarray(qrows).view(np.int16)).view(torch.bfloat16).to(dev)
    wpr = wl.L // 32
    masks = torch.zeros((wl.B, wl.Hq, nrows, wpr), dtype=torch.int32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for it in range(3 + iters):
        e0.record()
        ctx.select_prefill(layer, qd, row0, nrows, masks)
        e1.record()
        torch.cuda.synchronize()
        if it >= 3:
            ts.append(e0.elapsed_time(e1) * 1e3)
    if ctx.check_status():
        raise RuntimeError("device status flags set")
    us = statistics.median(ts)
    elems = wl.B * wl.Hq * sum(row0 + r + 1 for r in range(nrows))
    line = {"table": "prefill", "workload": wl.name, "kimp_gemm": dict(proj, frac_hbm=proj["gbs"] / peak),
            "select_prefill": {"rows": nrows, "row0": row0, "us_median": us, "us_p90": _pct(ts, 0.9),
                               "score_elements": elems, "elements_per_s": elems / (us * 1e-6),
                               "score_tflops": 2 * wl.d_imp * elems / (us * 1e-6) / 1e12,
                               "mask_bytes": masks.numel() * 4, "mask_gbs": masks.numel() * 4 / (us * 1e-6) / 1e9}}
    del ctx, bufs
    torch.cuda.empty_cache()
    return line


def _table_shard(wl, ranks_list, dev, iters, flush_buf, variant=None):
    """Sequence-sharded decode of one layer with R ranks emulated on this GPU
    in lock step (each rank its own context and caches, ranks in token
    order, the last one appending).  Per rank: the device time of its own
    kernels between the exchanges (median over steps); the exchanges, done
    here by in-process copies, are excluded and reported as bytes, since
    across GPUs they are NCCL collectives over NVLink."""
    import torch
    from query_aware_sparse_decode_b200 import synth as S
    from query_aware_sparse_decode_b200 import tb as TB
    from query_aware_sparse_decode_b200.shard import ShardBuffers, exchange_in_process, sel_rows, shard_step
    variant = TB.TB_BUTLER if variant is None else variant
    L0 = wl.L - 1
    max_len = (wl.L + 1 + 255) // 256 * 256
    full, bufs, _ = build(wl, max_len, dev, variant)
    k_full, v_full, kimp_full, w = bufs[0]

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    kn, vn = S.kv_new(wl, 0)
    kn, vn, qq, qi = bf(kn), bf(vn), bf(S.query(wl, 0)), bf(S.q_imp(wl, 0))
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    rows_out = []
    for R in ranks_list:
        per = (L0 + R - 1) // R
        starts = [r * per for r in range(R)]
        ranks = []
        for r in range(R):
            t0 = starts[r]
            n = (starts[r + 1] if r + 1 < R else L0) - t0
            cap = (n + 2 + 255) // 256 * 256
            cfg = TB.make_config(1, wl.B, wl.Hq, wl.Hkv, wl.D, wl.d_imp, wl.G, cap, "bf16", wl.keep_pct, wl.sink,
                                 wl.window, dense_layers=(), variant=variant)
            ctx = TB.Context(cfg, dev)
            k = torch.zeros((wl.B, wl.Hkv, cap, wl.D), dtype=torch.bfloat16, device=dev)
            v = torch.zeros_like(k)
            k[:, :, :n] = k_full[:, :, t0:t0 + n]
            v[:, :, :n] = v_full[:, :, t0:t0 + n]
            kimp = TB.kimp_cache(cfg, dev)
            ctx.bind_layer(0, k, v, kimp, w)
            ctx.set_seq_lens(0, [n] * wl.B)
            ctx.project_kimp(0, 0, n)
            ranks.append((ctx, n, t0, ShardBuffers(cfg, R, dev), (k, v, kimp)))
        stream = torch.cuda.current_stream(dev)
        per_rank = [[] for _ in range(R)]
        for it in range(3 + iters):
            for ctx, n, _, _, _ in ranks:
                ctx.set_seq_lens(0, [n] * wl.B)
            if flush_buf is not None:
                flush_buf.add_(1)
                flush_buf.view(torch.float32)[: 64 << 20].sum()
            steps = [shard_step(ctx, 0, r, R, t0, [wl.L] * wl.B, qq, qi, out, sb,
                                kn if r == R - 1 else None, vn if r == R - 1 else None, stream)
                     for r, (ctx, _, t0, sb, _) in enumerate(ranks)]
            evs = [[] for _ in range(R)]
            # the host issues the ranks' calls one by one; a device-side wait
            # queued first lets all of them be enqueued before the GPU reaches
            # them, so the events time the kernels and not the issuing
            torch.cuda._sleep(100_000_000)
            while True:
                ops = []
                for r, st in enumerate(steps):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    ops.append(next(st, None))
                    e1.record(stream)
                    evs[r].append((e0, e1))
                if all(o is None for o in ops):
                    break
                exchange_in_process(ops)
            torch.cuda.synchronize()
            for ctx, _, _, _, _ in ranks:
                if ctx.check_status():
                    raise RuntimeError("device status flags set")
            if it >= 3:
                for r in range(R):
                    per_rank[r].append(sum(a.elapsed_time(b) for a, b in evs[r]) * 1e3)
        med = [statistics.median(x) for x in per_rank]
        nrow = wl.B * sel_rows(ranks[0][0].cfg)
        part = wl.B * wl.Hq * (wl.D + 1) * 4
        rows_out.append({"ranks": R, "tokens_per_rank": [n for _, n, _, _, _ in ranks],
                         "us_per_rank": [round(x, 1) for x in med], "us_slowest_rank": round(max(med), 1),
                         "exchange_bytes_per_rank": {"hist_sum_2x": 2 * nrow * 2048 * 4,
                                                     "hist_gather": R * nrow * 2048 * 4,
                                                     "partials_gather": R * part}})
        del ranks
        torch.cuda.empty_cache()
    return {"table": "sequence_sharded", "workload": wl.name, "variant": _variant_name(variant),
            "emulated_on": "one GPU, ranks in lock step, calls enqueued behind a device wait",
            "rows": rows_out}


def config_rows(dev, iters, peak, n_layers_prefill=32):
    """The rows of the other workloads carried in the default bench line:
    the 8B-shaped single layer at L=32768 (50 % and dense), the prefill
    importance path (K_imp GEMM over 32 layers and the 1024-row causal
    selection) and the long-context sweep at L = 131072 and 262144 for the
    TokenButler and soft-voting variants at 10/30/50 %.  Per row: median
    per-kernel times of 20 single cold-L2 decode steps and the fraction of
    the HBM peak reached by the first pass (score, or soft-vote logits) plus
    the attention."""
    import torch
    from query_aware_sparse_decode_b200 import synth as S
    from query_aware_sparse_decode_b200 import tb as TB
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    cases = [(S.LLAMA8B_L32K, TB.TB_BUTLER), (S.LLAMA8B_L32K.with_(keep_pct=100), TB.TB_BUTLER)]
    for L in (131072, 262144):
        for P in S.SWEEP_KEEP:
            cases += [(S.sweep(L, P), TB.TB_BUTLER), (S.sweep(L, P), TB.TB_SOFTVOTE)]
    rows = []
    for wl, variant in cases:
        line = _table_case(wl, variant, dev, iters, flush_buf, peak, hot_l2=False)
        t, rt = line["us_cold_l2"], line["rates_cold_l2"]
        bt = line["us_batched"]
        rows.append({"workload": line["workload"], "variant": line["variant"], "L": line["L"],
                     "keep_pct": line["keep_pct"], "dense": line["dense"],
                     "us": {k: round(v, 2) for k, v in bt.items()},
                     "first_pass_bytes": line["first_pass_bytes"], "attn_bytes": line["attn_bytes"],
                     "pair_frac": (round(line["batched_pair_frac"], 4) if line["batched_pair_frac"] is not None
                                   else None),
                     "attn_frac": round(line["batched_attn_frac"], 4),
                     "us_traced": {k: round(t[k], 2) for k in ("score", "select", "attn", "combine", "total")},
                     "pair_frac_traced": (round(rt["score_plus_attn_frac"], 4) if "score_plus_attn_frac" in rt
                                          else None),
                     "attn_frac_traced": round(rt["attn_frac"], 4)})
    del flush_buf
    torch.cuda.empty_cache()
    pf = _table_prefill(dev, iters, peak, n_layers_prefill)
    prefill = {"kimp_gemm_us_per_layer": round(pf["kimp_gemm"]["us_per_layer"], 2),
               "kimp_gemm_frac_hbm": round(pf["kimp_gemm"]["frac_hbm"], 4),
               "kimp_gemm_tflops": round(pf["kimp_gemm"]["tflops"], 1),
               "select_rows_us": round(pf["select_prefill"]["us_median"], 1),
               "select_rows_elements_per_s": pf["select_prefill"]["elements_per_s"]}
    return {"decode_rows": rows, "prefill": prefill, "peak_gbs": peak,
            "timing": ("us / pair_frac / attn_frac: per call through the C ABI (score or soft-vote logits + reduce; "
                       "selection; attention + combine; the fused step), L2 cold (a 256 MB read before each call), "
                       "launches queued back to back so that no launch gap is counted: 10 (read, call) pairs minus "
                       "10 reads, median of 5; us_traced / pair_frac_traced: the fused step's segments between "
                       "trace events (each segment also holds the gap of its launch behind an event), median of "
                       "single steps, L2 flushed before each (512 MB write, 256 MB read)")}


def kernel_table(args):
    """Per-kernel times for the workloads beside the step benchmark: the
    8B-shaped L=32768 case (50 % and dense), the long-context sweep of both
    variants and the prefill importance path.  Prints one JSON line per row."""
    import torch
    from query_aware_sparse_decode_b200 import synth as S
    from query_aware_sparse_decode_b200 import tb as TB
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, _ = read_peak()
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    cases = [(S.LLAMA8B_L32K, TB.TB_BUTLER), (S.LLAMA8B_L32K.with_(keep_pct=100), TB.TB_BUTLER)]
    for L in S.SWEEP_LENGTHS:
        for P in S.SWEEP_KEEP:
            cases.append((S.sweep(L, P), TB.TB_BUTLER))
            cases.append((S.sweep(L, P), TB.TB_SOFTVOTE))
            cases.append((S.sweep(L, P), TB.TB_BUTLER_GROUP))
    import re
    pick = re.compile(args.table_only) if args.table_only else None
    for wl, variant in cases:
        name = f"{wl.name}_{_variant_name(variant)}"
        if pick is None or pick.search(name):
            print(json.dumps(_table_case(wl, variant, dev, args.table_iters, flush_buf, peak)), flush=True)
    if pick is None or pick.search(S.PREFILL_L32K.name):
        print(json.dumps(_table_prefill(dev, args.table_iters, peak, args.layers)), flush=True)
    for L in (131072, 262144):
        wl = S.sweep(L, 30)
        if pick is None or pick.search(f"shard_{wl.name}"):
            print(json.dumps(_table_shard(wl, (1, 2, 4, 8), dev, args.table_iters, flush_buf)), flush=True)


# ----------------------------------------------------------------------- main
def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if args.table:
        if rank == 0:
            kernel_table(args)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    if args.shard:
        shard_arm(args, rank, world, local_rank)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    r = gpu_arm(args, rank, world, local_rank)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(r["wl"], args.cpu_seconds, group=args.variant == "group", kimp=args.kimp)
    extra = None
    if rank == 0 and world == 1 and not args.no_config_rows:
        import torch
        dev = torch.device("cuda", local_rank)
        clk = ClockSampler(gpu_ident(dev, local_rank))
        clk.start()
        extra = config_rows(dev, args.table_iters, r["peak"])
        extra["clocks"] = clk.stop()
    if rank == 0:
        wl = r["wl"]
        avg = r["avg"]
        attn_launch_bytes = r["union_bytes"]
        line = {
            "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "layers": wl.n_layers, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv,
                       "D": wl.D, "d_imp": wl.d_imp, "G": wl.G, "L": wl.L, "keep_pct": wl.keep_pct,
                       "sink": wl.sink, "window": wl.window, "dense_layers": list(wl.dense_layers),
                       "selection": "per_kv_group" if args.variant == "group" else "per_query_head",
                       "kv_layout": f"paged, {args.page_size}-token pages" if args.page_size else "dense",
                       "kimp_cache": args.kimp,
                       "reuse": (None if not args.reuse else
                                 {"tau,interval,radius": args.reuse, "drift": args.drift,
                                  "note": "the length advances one token per step; scored and attended "
                                          "counts are those of a fresh step at L"}),
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (caches of all layers, no flush)"},
            "us_per_layer": r["ms_step"] * 1e3 / wl.n_layers,
            "tokens_scored_per_step": r["scored"], "tokens_attended_per_step": r["attended"],
            "hbm_gbs_step": r["step_bytes"] / (r["ms_step"] * 1e-3) / 1e9,
            "roofline": {"kernel": "butler_sparse_attn (sparse layers)", "bound": "hbm",
                         "achieved": r["attn_gbs"], "peak": r["peak"], "unit": "GB/s",
                         "frac": (r["attn_gbs"] / r["peak"]) if r["attn_gbs"] else None,
                         "traffic": (attn_traffic_per_row() * r["union_bytes"] / 512
                                     if attn_traffic_per_row() else None),
                         "bytes_per_launch": attn_launch_bytes, "peak_source": r["peak_src"]},
            "roofline_score_plus_attn": {"achieved": r["pair_gbs"], "peak": r["peak"], "unit": "GB/s",
                                         "frac": (r["pair_gbs"] / r["peak"]) if r["pair_gbs"] else None},
            "roofline_score": {"achieved": r["score_gbs"], "peak": r["peak"], "unit": "GB/s",
                               "frac": (r["score_gbs"] / r["peak"]) if r["score_gbs"] else None,
                               "bytes_per_launch": r["kimp_bytes"]},
            "kernel_us": avg,
            "prefill_kimp": dict(r["proj"], frac_hbm=r["proj"]["gbs"] / r["peak"]),
            "union_rows_per_layer": (sum(r["urows"].values()) / max(len(r["urows"]), 1)),
            "gpu_launches": r["launches"],
            "clocks": r["clk"],
            "e2e": r["e2e"],
            "cpu_baseline": cpu,
            "config_rows": extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
