"""Benchmark of the fused decode-GEMM path on one Llama-3.1-8B-shaped gate
projection W[14336, 4096] (BF16, N(0, 0.02) with a 0.1% t_3 tail) at batch 1.

One step = the whole per-call hot path over one batch:
  uw_decode_full, uw_decode_exponent, uw_transcode_palette, and
  uw_gemm through the four pipelines (full, exponent, transcode, direct
  palette) with x[1, 4096].
value = effective BF16 weight bytes delivered per second over the step
(7 x 2*N*K bytes per step / step time), whole job (all ranks).
The line also carries a batch sweep outside the timed step: the tensor-core
GEMM (direct palette, exponent pipeline, dense BF16) at M = 16 ... 1024 on
the same projection, each timed alone over rotated copies.

Inputs larger than L2: four compressed copies of W (~110 MB each) are
rotated so that an op never finds its inputs left in L2 by the previous use.
--impl reference times the CPU oracle (plain C) on a bounded row sample of the
same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused decode-GEMM eff. weight GB/s & TFLOP/s, % roofline, batch 1–1024"
N_W, K_W, M_X = 14336, 4096, 1
OPS = ["decode_full", "decode_exponent", "transcode", "gemm_full", "gemm_exponent", "gemm_transcode",
       "gemm_direct_palette"]
WORKLOAD = "gate projection W[14336,4096] bf16 N(0,0.02)+0.1% t3 tail, x[1,4096]; decode x3 + 4 pipelines"
OP_BURST = 8      # launches per graph when one op is timed alone


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # raw samples: $UW_CLOCKS_DIR if set, else the system temp directory
        import tempfile
        d = os.environ.get("UW_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, f"uw_bench_clocks_gpu{index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def mark(self, which: str):
        setattr(self, which, datetime.datetime.now())

    def summary(self):
        """Median SM clock and active throttle reasons over the samples taken
        between mark('t0') and mark('t1')."""
        try:
            rows = [[c.strip() for c in l.split(",")] for l in open(self.path).read().strip().splitlines()
                    if l.strip()]
        except Exception:
            rows = []
        t0, t1 = getattr(self, "t0", None), getattr(self, "t1", None)
        sel = []
        for r in rows:
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f")
            except Exception:
                continue
            if t0 is None or t1 is None or t0 <= ts <= t1:
                sel.append(r)
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = sorted(float(r[1]) for r in sel)
        mx = max(float(r[2]) for r in sel)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in sel for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": reasons, "samples": len(sel)}


def _dist(backend: str = "nccl"):
    """One process per GPU under torchrun: (dist module or None, rank, world,
    local rank).  The path does not shard, so ranks are independent replicas
    that meet only for the barriers around the timed region and the
    max-over-ranks reduction of its device time."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dist, int(os.environ["RANK"]), ws, int(os.environ.get("LOCAL_RANK", "0"))
    return None, 0, 1, 0


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's value (every rank gets it)."""
    if not dist:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)
# ---------------------------------------------------------------------------
_sample_cache = {}


def oracle_step_sample(rows: int = 256):
    """Runs the oracle's version of one step on `rows` rows of the workload:
    Huffman decode -> full / exponent / transcode, then the reference product
    for each of the four pipelines.  Returns (seconds, weights processed)."""
    import synthetic as S
    from oracle import oracle as O
    if rows not in _sample_cache:
        _sample_cache[rows] = S.gate_projection()[:rows].copy()
    W = _sample_cache[rows]
    x = S.activations(M_X, K_W, seed=1 + S.X_SEED_OFFSET)
    b = O.compress(W)
    t0 = time.perf_counter()
    Wd = O.decode_full(b)                 # decode_full
    O.decode_exponent(b)                  # decode_exponent
    O.transcode(b)                        # transcode
    for _ in range(4):                    # four pipelines: decode form + product
        O.decode_exponent(b)
        O.gemm(x, Wd, "f32")
    dt = time.perf_counter() - t0
    return dt, W.size


def cpu_baseline(rows: int = 256):
    dt, nw = oracle_step_sample(rows)
    eff = len(OPS) * 2.0 * nw / dt / 1e9
    return {"value": eff, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} of 14336 rows ({nw} weights), one step: decode x3 + 4 x (decode + GEMV), "
                      f"single thread, {dt:.3f} s"}


def run_reference(args):
    # the oracle runs on rank 0 only; other ranks exit at once (no process
    # group: they exchange nothing)
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    rows = 256
    for _ in range(args.warmup):
        oracle_step_sample(rows)
    tot = 0.0
    nw = 0
    for _ in range(args.steps):
        dt, nw = oracle_step_sample(rows)
        tot += dt
    value = len(OPS) * 2.0 * nw * args.steps / tot / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "oracle_rows_per_step": rows, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{rows} of 14336 rows per step, single thread"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_stack(args):
    """The 32-layer stack of Llama-3.1-8B-shaped MLP weights (synthetic, a
    per-layer seed and std): every gate, up and down matrix compressed and
    kept resident, the total footprint per form against BF16, and the
    autotuner's plan (pipeline and decoder SM split per projection and batch
    size, measured on layer 0) with the measured time of one layer's MLP
    matmuls.  Prints one JSON line; not part of the timed benchmark."""
    import numpy as np
    import torch
    import decode_gemm_bf16_b200 as uw
    import synthetic as S

    dev = torch.device("cuda", 0)
    Ms = [1, 8, 64, 256, 1024]
    t_start = time.time()
    blobs, bf16_bytes, huff, pal, devb = [], 0, 0, 0, 0
    for layer in range(args.layers):
        for W in S.stack_layer(layer):
            Wd = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
            b = uw.uw_compress(Wd)
            del Wd
            info = b.info
            bf16_bytes += 2 * W.size
            huff += info["bytes_huffman_form"]
            pal += info["bytes_palette_form"]
            devb += info["device_bytes"]
            blobs.append(b)
    torch.cuda.synchronize()
    t_compress = time.time() - t_start
    proj = blobs[:3]
    Xs = [torch.from_numpy(S.activations(max(Ms), b.info["K"], seed=7 + i).view(np.int16)).to(dev).view(torch.bfloat16)
          for i, b in enumerate(proj)]
    Ys = [torch.empty(max(Ms), b.info["N"], dtype=torch.bfloat16, device=dev) for b in proj]
    need = max(uw.uw_gemm_workspace(b, max(Ms), p, sm_dec=sd) for b in proj for p in uw.PIPELINES for sd in (0, 296))
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    plan = uw.uw_autotune(proj, Ms, Xs, Ys, ws, reps=5)
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during the stack run")
    layer_us = {str(M): sum(e["us"] for e in plan if e["M"] == M) for M in Ms}
    flops = {str(M): 2.0 * M * sum(b.info["N"] * b.info["K"] for b in proj) for M in Ms}
    line = {"stack": {"layers": args.layers, "matrices": len(blobs), "weights": bf16_bytes // 2,
                      "bf16_bytes": bf16_bytes, "huffman_form_bytes": huff, "palette_form_bytes": pal,
                      "device_image_bytes": devb, "ratio_huffman_form": huff / bf16_bytes,
                      "ratio_palette_form": pal / bf16_bytes, "compress_s_incl_host_generation": t_compress},
            "plan_layer0": plan,
            "layer_mlp_us": layer_us,
            "layer_mlp_tflops": {M: flops[M] / (layer_us[M] * 1e-6) / 1e12 for M in layer_us}}
    print(json.dumps(line), flush=True)


def uw_gemv_serves():
    """Whether batch 1 on this projection runs the CUDA-core GEMV (the
    library's rule: fewer than half as many 128-row tiles as GEMM CTAs)."""
    import torch
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return 2 * ((N_W + 127) // 128) < sms


def batch_sweep(uw, torch, S, copies, dev, cap, capture, tc_peak, hbm_peak):
    """Tensor-core GEMM at larger batches on the same projection (outside the
    timed step): per M and pipeline, device time of one call (graph replays
    over the rotated copies), TFLOP/s against the measured dense BF16 peak
    and effective BF16 weight GB/s."""
    import numpy as np
    n = N_W * K_W
    Wd = torch.from_numpy(S.gate_projection().view(np.int16)).to(dev).view(torch.bfloat16)
    dense = [Wd] + [Wd.clone() for _ in range(3)]
    out = {}
    for M in (16, 64, 256, 1024):
        X = torch.from_numpy(S.activations(M, K_W, seed=M + S.X_SEED_OFFSET).view(np.int16)).to(dev).view(torch.bfloat16)
        Y = torch.empty(M, N_W, dtype=torch.bfloat16, device=dev)
        wsb = max([uw.uw_gemm_workspace(copies[0], M, p) for p in ("direct_palette", "exponent")] +
                  [uw.uw_dense_gemm_workspace(M, N_W, K_W)])
        ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        row = {}
        for name in ("direct_palette", "exponent", "dense"):
            if name == "dense":
                fns = [lambda w=w: uw.uw_dense_gemm(X, w, out=Y, ws=ws) for w in dense]
            else:
                fns = [lambda b=b, name=name: uw.uw_gemm(X, b, name, out=Y, ws=ws) for b in copies]
            with torch.cuda.stream(cap):
                for f in fns:
                    f()
            torch.cuda.synchronize()
            g = capture(lambda: [fns[i % len(fns)]() for i in range(OP_BURST)])
            for i in range(2):
                g.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 8
            a.record()
            for i in range(reps):
                g.replay()
            b.record()
            torch.cuda.synchronize()
            us = 1e3 * a.elapsed_time(b) / (reps * OP_BURST)
            tflops = 2.0 * M * n / (us / 1e6) / 1e12
            row[name] = {"us": us, "tflops": tflops, "tensor_frac": tflops / tc_peak,
                         "eff_weight_gbs": 2.0 * n / (us / 1e6) / 1e9}
            del g
        out[str(M)] = row
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during the batch sweep")
    return out


def run_gpu(args):
    import numpy as np
    import torch
    import decode_gemm_bf16_b200 as uw
    import synthetic as S

    dist, rank, world, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_peak, tc_peak, peak_kind = _peaks()

    W = S.gate_projection()
    x = S.activations(M_X, K_W, seed=1 + S.X_SEED_OFFSET)
    Wd = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
    copies = [uw.uw_compress(Wd) for _ in range(4)]
    del Wd
    info = copies[0].info
    n = N_W * K_W
    xd = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    wsb = max(uw.uw_gemm_workspace(copies[0], M_X, p) for p in uw.PIPELINES)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    out_full = torch.empty(N_W, K_W, dtype=torch.bfloat16, device=dev)
    out_e = torch.empty(n, dtype=torch.uint8, device=dev)
    out_i = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    Ys = [torch.empty(M_X, N_W, dtype=torch.bfloat16, device=dev) for _ in range(4)]
    stream = torch.cuda.current_stream()

    def op(k, blob, xin):
        if k == 0:
            uw.uw_decode_full(blob, out_full)
        elif k == 1:
            uw.uw_decode_exponent(blob, out_e)
        elif k == 2:
            uw.uw_transcode_palette(blob, out_i)
        else:
            uw.uw_gemm(xin, blob, k - 3, out=Ys[k - 3], ws=ws)

    nops = len(OPS)
    ncopy = len(copies)
    cap = torch.cuda.Stream(device=dev)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            fn()
        return g

    # every op once eagerly (sets kernel attributes), then one graph per
    # rotation of the weight copies: step r runs op k on copy (r + k) % 4
    with torch.cuda.stream(cap):
        for k in range(nops):
            op(k, copies[k % ncopy], xd)
    torch.cuda.synchronize()
    step_graphs = [capture(lambda r=r: [op(k, copies[(r + k) % ncopy], xd) for k in range(nops)])
                   for r in range(ncopy)]
    # per-op graphs: OP_BURST launches of one op over the rotated copies, so the
    # per-launch time is not inflated by the gap between graph launches
    op_graphs = [capture(lambda k=k: [op(k, copies[i % ncopy], xd) for i in range(OP_BURST)]) for k in range(nops)]

    # warm-up: W steps, and at least half a second of work so the clocks settle
    t_w = time.time()
    i = 0
    while i < max(3, args.warmup) or time.time() - t_w < 0.5:
        step_graphs[i % ncopy].replay()
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # ---- timed region: K steps (graph replays), device time with CUDA events
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        time.sleep(0.3)           # let the sampler start
        clk.mark("t0")
        t0.record(stream)
        for i in range(args.steps):
            step_graphs[i % ncopy].replay()
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark("t1")
    if dist:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if dist:
        ms = max_over_ranks(ms, dist, dev)
    # per-op device time: each op alone, rotated over the copies
    reps = max(10, min(100, args.steps // 20))
    per_op_ms = []
    for k in range(nops):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(2):
            op_graphs[k].replay()
        a.record(stream)
        for i in range(reps):
            op_graphs[k].replay()
        b.record(stream)
        torch.cuda.synchronize()
        per_op_ms.append(a.elapsed_time(b) / (reps * OP_BURST))
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during the timed region")
    sweep = batch_sweep(uw, torch, S, copies, dev, cap, capture, tc_peak, hbm_peak) if not args.no_sweep else None

    # ---- end to end: host x (pinned) -> device, the step, Y -> host (pinned)
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = [torch.empty(M_X, N_W, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    xdev = torch.empty_like(xd)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for k in range(nops):
        op(k, copies[k % ncopy], xdev)
    torch.cuda.synchronize()
    e0.record(stream)
    ctr = 0
    for i in range(args.steps):
        xdev.copy_(xh, non_blocking=True)
        for k in range(nops):
            op(k, copies[ctr % ncopy], xdev)
            ctr += 1
        for j in range(4):
            yh[j].copy_(Ys[j], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if dist:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)

    # ---- numbers
    eff_bytes_step = nops * 2.0 * n
    value = world * eff_bytes_step * args.steps / (ms / 1e3) / 1e9
    e2e = world * eff_bytes_step * args.steps / (e2e_ms / 1e3) / 1e9
    sec = info["sections"]
    stream_b = sec["stream"][1] + sec["chunk_off"][1] + sec["seg_rel"][1]
    vstore = sec["vbits"][1] + sec["vpre"][1] + sec["vexp"][1]
    xb, yb = M_X * K_W * 2, M_X * N_W * 2
    # algorithmic bytes per launch of each single-kernel op (what must move)
    alg = {
        "decode_full": stream_b + vstore + n + 2 * n,
        "decode_exponent": stream_b + vstore + n,
        "transcode": stream_b + n // 2,
        "gemm_direct_palette": n + n // 2 + vstore + xb + yb + (0 if uw_gemv_serves() else sec["vcol"][1]),
    }
    kernel_of = {"decode_full": "k_decode<full>", "decode_exponent": "k_decode<exponent>",
                 "transcode": "k_decode<transcode>",
                 "gemm_direct_palette": "k_gemv<palette, M=1>" if uw_gemv_serves() else "k_gemm_recon<palette>"}
    breakdown = {}
    for k, name in enumerate(OPS):
        d = {"us": 1e3 * per_op_ms[k], "eff_weight_gbs": 2.0 * n / (per_op_ms[k] / 1e3) / 1e9,
             "tflops": (2.0 * M_X * n / (per_op_ms[k] / 1e3) / 1e12) if name.startswith("gemm") else None}
        if name in alg:
            d["alg_bytes"] = alg[name]
            d["alg_gbs"] = alg[name] / (per_op_ms[k] / 1e3) / 1e9
            d["hbm_frac"] = d["alg_gbs"] / hbm_peak
        breakdown[name] = d
    # dominant single-kernel op: the decode_full kernel also runs inside the
    # full pipeline, the palette GEMM inside the transcode pipeline
    share = {"decode_full": per_op_ms[0] * 2, "decode_exponent": per_op_ms[1] * 2,
             "transcode": per_op_ms[2] * 2, "gemm_direct_palette": per_op_ms[6] * 2}
    dom = max(share, key=share.get)
    dom_ms = per_op_ms[OPS.index(dom)]
    achieved = alg[dom] / (dom_ms / 1e3) / 1e9
    # DRAM bytes per launch from the committed ncu capture, only while the
    # kernel is the one that capture measured (same code hash of its
    # translation unit: sources without comments, plus build flags)
    traffic = None
    tp = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tp):
        try:
            from decode_gemm_bf16_b200 import build as uwbuild
            tj = json.load(open(tp))
            ent = tj["bytes_per_launch"].get(kernel_of[dom])
            if ent and ent.get("code_hash") == uwbuild.kernel_code_hash(kernel_of[dom]):
                traffic = ent["bytes"]
        except Exception:
            traffic = None
    launches_per_step = 3 + 2 + 2 + 2 + 1
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_X, "N": N_W, "K": K_W, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2: 4 rotating compressed copies",
                   "ratio_huffman_form": info["bytes_huffman_form"] / (2 * n),
                   "ratio_palette_form": info["bytes_palette_form"] / (2 * n),
                   "mean_code_bits": info["mean_code_len"]},
        "roofline": {"bound": "hbm", "kernel": kernel_of[dom], "achieved": achieved, "peak": hbm_peak,
                     "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)", "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic},
        "breakdown": breakdown,
        "batch_sweep": sweep,
        "e2e": {"value": e2e, "unit": "GB/s", "h2d_bytes_per_step": xb, "d2h_bytes_per_step": 4 * yb},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-sweep", action="store_true", help="skip the larger-batch GEMM sweep")
    ap.add_argument("--stack", action="store_true",
                    help="compress the synthetic 32-layer MLP stack, report footprint and the autotuned plan")
    ap.add_argument("--layers", type=int, default=32, help="layers for --stack")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.stack:
        run_stack(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
