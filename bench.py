"""Benchmark of the fused decode-GEMM path on the 32-layer stack of
Llama-3.1-8B-shaped MLP weights (synthetic: gate/up W[14336,4096], down
W[4096,14336] per layer, BF16 N(0, sigma_l) with a 0.1% t_3 tail, sigma_l ~
U(0.015, 0.03)), every matrix compressed and resident on the GPU.

One step = one pass over all 96 matrices at each batch size M in
{1, 8, 64, 256, 1024}: Y = X . W^T through uw_gemm with UW_PIPE_AUTO, i.e.
the pipeline, matmul variant and decoder split the autotuner (§自動調優機制)
chose for that projection and batch on this GPU.  The activations are fixed
synthetic X[M, 4096] (gate, up) and X[M, 14336] (down).
value = effective BF16 weight bytes per second over the step (5 x 96
matrices x 2*N*K bytes per step / step time), whole job (all ranks).

Inputs are larger than L2: consecutive calls use different matrices, so no
weight is read from L2 left by the previous use.

The line also carries, outside the timed step: per (projection, M) the time
of one call (the plan's choice, rotated over the layers) with its compressed
GB/s, TFLOP/s, roofline fraction and slowdown against the library's own
dense BF16 GEMM; the compressed footprint of the stack per form; the
decoders and the five pipelines at batch 1 on the gate projection; the
decoder/matmul SM split swept on the down projection at M = 256 and 1024;
one MLP layer with gate+up in one launch (SwiGLU epilogue) feeding down; and
the stack run as a sequence of hard (Huffman) and easy (palette) layers.

--impl reference times the CPU oracle (plain C) on a bounded row sample of the
same step and prints the same metric.
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
MS = [1, 8, 64, 256, 1024]
PROJ = ["gate", "up", "down"]
SHAPES = {"gate": (14336, 4096), "up": (14336, 4096), "down": (4096, 14336)}
WORKLOAD = ("32-layer Llama-3.1-8B-shaped MLP stack (gate/up W[14336,4096], down W[4096,14336]; bf16 "
            "N(0,s_l)+0.1% t3 tail, s_l~U(0.015,0.03)); one step = all 96 matrices at each batch "
            "M in {1,8,64,256,1024}, autotuned plan (UW_PIPE_AUTO)")
OP_BURST = 8      # launches per graph when one op is timed alone
ORACLE_ROWS_CPU = 256      # rows per projection in the CPU baseline sample
ORACLE_ROWS_REF = 16       # rows per projection in one step of --impl reference


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return (float(d.get("hbm_gbs", 6650.0)), float(d.get("bf16_tflops", 1590.0)),
                float(d.get("bf16_tflops_sustained", 1400.0)), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


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
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
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
        try:
            pw = sorted(float(r[3]) for r in sel)
            power = pw[len(pw) // 2]
        except Exception:
            power = None
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": reasons, "samples": len(sel),
                "power_w_median": power}


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


def _oracle_sample(rows: int):
    """`rows` rows of each projection of layer 0's shape and distribution
    (host recipe), compressed by the oracle; activations per projection and M."""
    if rows not in _sample_cache:
        import synthetic as S
        from oracle import oracle as O
        sd = float(S.layer_stds()[0])
        sample = []
        for j, name in enumerate(PROJ):
            K = SHAPES[name][1]
            Wr = S.weight_with_tail(rows, K, seed=1000 + j, std=sd)
            X = {M: S.activations(M, K, seed=7 + j + M) for M in MS}
            sample.append((name, O.compress(Wr), X))
        _sample_cache[rows] = sample
    return _sample_cache[rows]


def oracle_step_sample(rows: int, threads: int):
    """The oracle's version of one step on `rows` rows of every projection of
    layer 0, at each batch size: rebuild the rows from their compressed form
    (direct palette: palette lookup, verbatim groups, merge) and form
    X . W^T, in `threads` threads over row blocks.  Returns (seconds,
    weights processed, flops)."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as O
    sample = _oracle_sample(rows)
    blocks = []
    for name, b, X in sample:
        for M in MS:
            blocks.append((b, X[M]))
    nw = sum(b["N"] * b["K"] for _, b, _ in sample) * len(MS)
    flops = sum(2.0 * M * b["N"] * b["K"] for _, b, _ in sample for M in MS)

    def one(item):
        b, x = item
        W = O.decode_full(b)
        O.gemm(x, W, "f32")

    t0 = time.perf_counter()
    if threads <= 1:
        for it in blocks:
            one(it)
    else:
        # split every block's rows so all threads have work
        parts = []
        import numpy as np
        for b, x in blocks:
            W = O.decode_full(b)
            step = max(1, -(-W.shape[0] // threads))
            for r0 in range(0, W.shape[0], step):
                parts.append((x, np.ascontiguousarray(W[r0:r0 + step])))
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda p: O.gemm(p[0], p[1], "f32"), parts))
    dt = time.perf_counter() - t0
    return dt, nw, flops


def cpu_baseline():
    cores = os.cpu_count() or 1
    _oracle_sample(ORACLE_ROWS_CPU)
    dt1, nw, fl = oracle_step_sample(ORACLE_ROWS_CPU, 1)
    dtn, _, _ = oracle_step_sample(ORACLE_ROWS_CPU, cores)
    return {"value": 2.0 * nw / dtn / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "single_thread_value": 2.0 * nw / dt1 / 1e9, "tflops_all_cores": fl / dtn / 1e12,
            "sample": f"{ORACLE_ROWS_CPU} rows of each of gate, up and down (layer 0 shapes and std), at each M in {MS}: "
                      f"rebuild rows from the palette form + X.W^T in fp32 ({nw} weights x batch); "
                      f"{cores} threads {dtn:.2f} s, 1 thread {dt1:.2f} s"}


def run_reference(args):
    # the oracle runs on rank 0 only; other ranks exit at once (no process
    # group: they exchange nothing)
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    rows = ORACLE_ROWS_REF
    _oracle_sample(rows)
    for _ in range(args.warmup):
        oracle_step_sample(rows, cores)
    tot, nw = 0.0, 0
    for _ in range(args.steps):
        dt, nw, _ = oracle_step_sample(rows, cores)
        tot += dt
    value = 2.0 * nw * args.steps / tot / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "oracle_rows_per_projection_per_step": rows, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} rows of each of gate, up and down at each M in {MS} "
                                       f"per step, {cores} threads"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def _alg_bytes(info, pipeline, M, gemv):
    """Bytes the method must move for one call (what a perfect kernel reads
    and writes): the compressed planes it reads, intermediate planes written
    and read back, activations and outputs."""
    sec = info["sections"]
    n = info["N"] * info["K"]
    stream_b = sec["stream"][1] + sec["chunk_off"][1] + sec["seg_rel"][1]
    vstore = sec["vbits"][1] + sec["vpre"][1] + sec["vexp"][1]
    vcol = 0 if gemv else sec["vcol"][1]
    xy = 2 * M * (info["N"] + info["K"])
    if pipeline == "direct_palette":
        return n + n // 2 + vstore + vcol + xy
    if pipeline == "transcode":
        return (stream_b + n // 2) + (n + n // 2 + vstore + vcol + xy)
    if pipeline == "exponent":
        return (stream_b + vstore + n) + (2 * n + xy)
    if pipeline == "fused_huffman":
        return stream_b + n + vstore + xy
    return (stream_b + vstore + n + 2 * n) + (2 * n + xy)   # full


def _kernel_name(pipeline, gemv):
    if pipeline == "fused_huffman":
        return "k_fused_huffman"
    if pipeline == "full":
        return "k_gemv<dense, M=1>" if gemv else "k_gemm_dense"
    src = "exponent" if pipeline == "exponent" else "palette"
    return f"k_gemv<{src}, M=1>" if gemv else f"k_gemm_recon<{src}>"


def run_gpu(args):
    import numpy as np
    import torch
    import decode_gemm_bf16_b200 as uw
    import synthetic as S

    dist, rank, world, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_peak, tc_burst, tc_sust, peak_kind = _peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    L = args.layers
    t_start = time.time()

    # ---- the stack: draw, compress, keep resident (dense copies of the first
    # few layers stay too, for the dense baseline)
    n_dense = min(4, L)
    blobs = [[None] * 3 for _ in range(L)]
    dense = [[None] * 3 for _ in range(n_dense)]
    foot = {"bf16": 0, "huffman_form": 0, "palette_form": 0, "device_image": 0}
    per_proj_ratio = {p: [0, 0, 0] for p in PROJ}
    for layer in range(L):
        mats = S.stack_layer_device(layer, dev)
        for j, W in enumerate(mats):
            b = uw.uw_compress(W)
            blobs[layer][j] = b
            info = b.info
            nbytes = 2 * W.numel()
            foot["bf16"] += nbytes
            foot["huffman_form"] += info["bytes_huffman_form"]
            foot["palette_form"] += info["bytes_palette_form"]
            foot["device_image"] += info["device_bytes"]
            r = per_proj_ratio[PROJ[j]]
            r[0] += nbytes
            r[1] += info["bytes_huffman_form"]
            r[2] += info["bytes_palette_form"]
            if layer < n_dense:
                dense[layer][j] = W
        del mats
    torch.cuda.synchronize()
    t_compress = time.time() - t_start

    # activations per (projection input width, M); outputs per (projection, M)
    Xg = {M: S.activations_device(M, 4096, seed=17 + M, device=dev) for M in MS}
    Xd = {M: S.activations_device(M, 14336, seed=29 + M, device=dev) for M in MS}
    Xof = {"gate": Xg, "up": Xg, "down": Xd}
    Y = {(p, M): torch.empty(M, SHAPES[p][0], dtype=torch.bfloat16, device=dev) for p in PROJ for M in MS}

    # ---- autotune on the first layers (each layer is a copy of the shapes)
    n_copies = min(4, L)
    tune_blobs = [blobs[c][j] for c in range(n_copies) for j in range(3)]
    Mmax = max(MS)
    tX = [Xg[Mmax], Xg[Mmax], Xd[Mmax]]
    tY = [Y[(p, Mmax)] for p in PROJ]
    need = max(uw.uw_gemm_workspace(b, Mmax, p, sm_dec=sd) for b in blobs[0] for p in uw.PIPELINES
               for sd in (0, sms // 2, sms, 2 * sms))
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    t_tune = time.time()
    plan_entries = uw.uw_autotune(tune_blobs, MS, tX, tY, ws, reps=3, copies=n_copies)
    t_tune = time.time() - t_tune
    plan = uw.Plan(plan_entries)
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during autotuning")
    choice = {(PROJ[e["projection"]], e["M"]): e for e in plan_entries}

    def call(p, M, layer, xin=None, yout=None):
        j = PROJ.index(p)
        uw.uw_gemm(xin if xin is not None else Xof[p][M], blobs[layer][j], "auto",
                   out=yout if yout is not None else Y[(p, M)], ws=ws, plan=plan, projection=j)

    def step():
        for M in MS:
            for layer in range(L):
                for p in PROJ:
                    call(p, M, layer)

    cap = torch.cuda.Stream(device=dev)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            fn()
        return g

    with torch.cuda.stream(cap):
        step()                       # eager once: kernel attributes, side streams
    torch.cuda.synchronize()
    step_graph = capture(step)
    launches_per_step = 0
    for M in MS:
        for p in PROJ:
            e = choice[(p, M)]
            per_call = 1 + (0 if e["pipeline"] == "direct_palette" else 1)
            launches_per_step += L * per_call

    # warm-up: W steps, and at least a second of work so the clocks settle
    t_w = time.time()
    i = 0
    while i < max(3, args.warmup) or time.time() - t_w < 1.0:
        step_graph.replay()
        i += 1
        torch.cuda.synchronize()
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # ---- timed region: K steps (graph replays), device time with CUDA events
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        time.sleep(0.3)           # let the sampler start
        clk.mark("t0")
        t0.record(stream)
        for i in range(args.steps):
            step_graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark("t1")
    if dist:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if dist:
        ms = max_over_ranks(ms, dist, dev)
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during the timed region")
    del step_graph

    def time_graph(g, launches, reps=5):
        for _ in range(2):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return 1e3 * a.elapsed_time(b) / (reps * launches)   # microseconds per launch

    # ---- per (projection, M): the plan's call alone, over all layers; the
    # dense baseline over the dense copies
    dense_ws = torch.zeros(max(uw.uw_dense_gemm_workspace(M, *SHAPES[p]) for p in PROJ for M in MS),
                           dtype=torch.uint8, device=dev)
    per = {}
    for p in PROJ:
        N, K = SHAPES[p]
        info = blobs[0][PROJ.index(p)].info
        for M in MS:
            g = capture(lambda p=p, M=M: [call(p, M, layer) for layer in range(L)])
            us = time_graph(g, L)
            del g
            nd = n_dense * max(1, OP_BURST // n_dense)
            gd = capture(lambda p=p, M=M: [uw.uw_dense_gemm(Xof[p][M], dense[i % n_dense][PROJ.index(p)],
                                                            out=Y[(p, M)], ws=dense_ws) for i in range(nd)])
            us_dense = time_graph(gd, nd)
            del gd
            e = choice[(p, M)]
            gemv = (e["variant"] == 2) or (e["variant"] == 0 and M == 1 and e["sm_dec"] == 0 and
                                            2 * ((N + 127) // 128) < (e["grid"] or sms))
            alg = _alg_bytes(info, e["pipeline"], M, gemv)
            flops = 2.0 * M * N * K
            gbs = alg / (us * 1e-6) / 1e9
            tfl = flops / (us * 1e-6) / 1e12
            per[f"{p}/M={M}"] = {
                "us": us, "pipeline": e["pipeline"], "variant": e["variant"], "sm_dec": e["sm_dec"],
                "grid": e["grid"], "split_k": e["split_k"], "kernel": _kernel_name(e["pipeline"], gemv),
                "alg_bytes": alg, "compressed_gbs": gbs, "eff_weight_gbs": 2.0 * N * K / (us * 1e-6) / 1e9,
                "tflops": tfl, "hbm_frac": gbs / hbm_peak, "tensor_frac": tfl / tc_burst,
                "roofline_frac": max(gbs / hbm_peak, tfl / tc_burst),
                "bound": "tensor" if tfl / tc_burst > gbs / hbm_peak else "hbm",
                "dense_us": us_dense, "slowdown_vs_dense": us / us_dense,
                "share_of_step": L * us / (1e3 * ms / args.steps)}
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set while timing single calls")

    # ---- the decoders and the four pipelines at batch 1 on the gate
    # projection (layers 0..3 rotated), and the SM split on the down projection
    ops = {}
    gate_blobs = [blobs[c][0] for c in range(n_copies)]
    ginfo = gate_blobs[0].info
    n = 14336 * 4096
    out_full = torch.empty(14336, 4096, dtype=torch.bfloat16, device=dev)
    out_e = torch.empty(n, dtype=torch.uint8, device=dev)
    out_i = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    sec = ginfo["sections"]
    stream_b = sec["stream"][1] + sec["chunk_off"][1] + sec["seg_rel"][1]
    vstore = sec["vbits"][1] + sec["vpre"][1] + sec["vexp"][1]
    dec_alg = {"decode_full": stream_b + vstore + 3 * n, "decode_exponent": stream_b + vstore + n,
               "transcode": stream_b + n // 2}
    dec_fn = {"decode_full": lambda b: uw.uw_decode_full(b, out_full),
              "decode_exponent": lambda b: uw.uw_decode_exponent(b, out_e),
              "transcode": lambda b: uw.uw_transcode_palette(b, out_i)}
    for name, fn in dec_fn.items():
        g = capture(lambda fn=fn: [fn(gate_blobs[i % n_copies]) for i in range(OP_BURST)])
        us = time_graph(g, OP_BURST)
        del g
        ops[name] = {"us": us, "alg_bytes": dec_alg[name], "alg_gbs": dec_alg[name] / (us * 1e-6) / 1e9,
                     "hbm_frac": dec_alg[name] / (us * 1e-6) / 1e9 / hbm_peak}
    for pipe in ["full", "exponent", "transcode", "direct_palette", "fused_huffman"]:
        g = capture(lambda pipe=pipe: [uw.uw_gemm(Xg[1], gate_blobs[i % n_copies], pipe, out=Y[("gate", 1)], ws=ws)
                                       for i in range(OP_BURST)])
        us = time_graph(g, OP_BURST)
        del g
        gemv = 2 * 112 < sms
        alg = _alg_bytes(ginfo, pipe, 1, gemv)
        ops[f"gemm_{pipe}"] = {"us": us, "alg_bytes": alg, "alg_gbs": alg / (us * 1e-6) / 1e9,
                               "hbm_frac": alg / (us * 1e-6) / 1e9 / hbm_peak,
                               "eff_weight_gbs": 2.0 * n / (us * 1e-6) / 1e9}
    sm_split = {}
    down_blobs = [blobs[c][2] for c in range(n_copies)]
    for M in (256, 1024):
        row = {}
        for pipe, sds in (("direct_palette", (0,)), ("exponent", (0, sms // 4, sms // 2, sms, 2 * sms))):
            for sd in sds:
                g = capture(lambda pipe=pipe, sd=sd, M=M: [
                    uw.uw_gemm(Xd[M], down_blobs[i % n_copies], pipe, out=Y[("down", M)], ws=ws, sm_dec=sd)
                    for i in range(n_copies)])
                us = time_graph(g, n_copies, reps=3)
                del g
                row[f"{pipe}/sm_dec={sd}"] = {"us": us, "tflops": 2.0 * M * 4096 * 14336 / (us * 1e-6) / 1e12}
        sm_split[f"M={M}"] = row
    # ---- one MLP layer with the real data flow: gate+up in one launch with
    # the SwiGLU epilogue, its output H feeding the down projection, against
    # the plan's separate gate, up and down calls (layers rotated)
    mlp = {}
    Hs = {M: torch.empty(M, 14336, dtype=torch.bfloat16, device=dev) for M in MS}
    sw_ws = torch.zeros(max(uw.uw_gemm_swiglu_workspace(blobs[0][0], blobs[0][1], M) for M in MS),
                        dtype=torch.uint8, device=dev)
    for M in MS:
        g = capture(lambda M=M: [(uw.uw_gemm_swiglu(Xg[M], blobs[l][0], blobs[l][1], out=Hs[M], ws=sw_ws),
                                  call("down", M, l, xin=Hs[M])) for l in range(L)])
        us_fused = time_graph(g, L)
        del g
        g = capture(lambda M=M: [uw.uw_gemm_swiglu(Xg[M], blobs[l][0], blobs[l][1], out=Hs[M], ws=sw_ws)
                                 for l in range(L)])
        us_sw = time_graph(g, L)
        del g
        sep = per[f"gate/M={M}"]["us"] + per[f"up/M={M}"]["us"] + per[f"down/M={M}"]["us"]
        mlp[f"M={M}"] = {"fused_layer_us": us_fused, "swiglu_gate_up_us": us_sw,
                         "separate_gate_up_us": per[f"gate/M={M}"]["us"] + per[f"up/M={M}"]["us"],
                         "separate_layer_us": sep, "speedup": sep / us_fused,
                         "swiglu_tflops": 2 * 2.0 * M * 14336 * 4096 / (us_sw * 1e-6) / 1e12}

    # ---- cross-layer hard/easy pipelining (§跨層管道化): the stack's
    # projections as one sequence, every layer easy (palette form), every
    # even layer hard (Huffman form, transcoded ahead on a side stream), or
    # every layer hard
    hard_easy = {}
    seq_ws = None
    for M in (1, 64, 256):
        row = {}
        for name, hard_of in (("all_easy", lambda l: False), ("alternate", lambda l: l % 2 == 0),
                              ("all_hard", lambda l: True)):
            items = [(blobs[l][j], Xof[p][M], Y[(p, M)], hard_of(l)) for l in range(L) for j, p in enumerate(PROJ)]
            need = uw.uw_sequence_workspace(items, M)
            if seq_ws is None or seq_ws.numel() < need:
                seq_ws = torch.zeros(need, dtype=torch.uint8, device=dev)
            for dec in ((0, sms) if name != "all_easy" else (0,)):
                g = capture(lambda items=items, dec=dec: uw.uw_gemm_sequence(items, M, dec_ctas=dec, ws=seq_ws))
                us = time_graph(g, L, reps=3)
                del g
                row[f"{name}/dec_ctas={dec}"] = {"us_per_layer": us}
        hard_easy[f"M={M}"] = row
    pal_b = foot["palette_form"] / L
    huf_b = foot["huffman_form"] / L
    hard_easy["footprint_ratio"] = {"all_easy": foot["palette_form"] / foot["bf16"],
                                    "alternate": (pal_b * (L // 2) + huf_b * (L - L // 2)) / foot["bf16"],
                                    "all_hard": foot["huffman_form"] / foot["bf16"]}
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set during the breakdowns")

    # ---- end to end: every step, the activations of every batch size are
    # copied from pinned host memory, the step runs through the public API
    # (eager calls, no graph), and every batch's last down-projection output
    # is copied back to pinned host memory
    xh = {(w, M): (Xg if w == 4096 else Xd)[M].cpu().pin_memory() for w in (4096, 14336) for M in MS}
    yh = {M: torch.empty(M, 4096, dtype=torch.bfloat16).pin_memory() for M in MS}
    xdev = {k: torch.empty_like(v, device=dev) for k, v in xh.items()}
    h2d = sum(v.numel() * 2 for v in xh.values())
    d2h = sum(v.numel() * 2 for v in yh.values())

    def e2e_step():
        for (w, M), t in xh.items():
            xdev[(w, M)].copy_(t, non_blocking=True)
        for M in MS:
            for layer in range(L):
                for p in PROJ:
                    call(p, M, layer, xin=xdev[(4096 if p != "down" else 14336, M)])
            yh[M].copy_(Y[("down", M)], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if dist:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)

    # ---- numbers
    weight_bytes_pass = sum(2 * SHAPES[p][0] * SHAPES[p][1] for p in PROJ) * L
    eff_bytes_step = weight_bytes_pass * len(MS)
    flops_step = sum(2.0 * M * SHAPES[p][0] * SHAPES[p][1] for p in PROJ for M in MS) * L
    ms_step = ms / args.steps
    value = world * eff_bytes_step / (ms_step / 1e3) / 1e9
    e2e = world * eff_bytes_step / (e2e_ms / 1e3) / 1e9
    # dominant kernel: the (projection, M) call with the largest share of the step
    dom_key = max(per, key=lambda k: per[k]["share_of_step"])
    d = per[dom_key]
    if d["bound"] == "tensor":
        roof = {"bound": "tensor", "kernel": d["kernel"], "call": dom_key, "achieved": d["tflops"],
                "peak": tc_burst, "peak_kind": f"{peak_kind} bf16_tflops (cuBLAS, burst; call timed alone)",
                "unit": "TFLOP/s", "frac": d["tflops"] / tc_burst,
                "frac_of_sustained": d["tflops"] / tc_sust}
    else:
        roof = {"bound": "hbm", "kernel": d["kernel"], "call": dom_key, "achieved": d["compressed_gbs"],
                "peak": hbm_peak, "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)", "unit": "GB/s",
                "frac": d["compressed_gbs"] / hbm_peak}
    roof["traffic"] = None
    tp = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tp):
        try:
            from decode_gemm_bf16_b200 import build as uwbuild
            tj = json.load(open(tp))
            ent = tj["bytes_per_launch"].get(f"{d['kernel']} {dom_key}")
            if ent and ent.get("code_hash") == uwbuild.kernel_code_hash(d["kernel"]):
                roof["traffic"] = ent["bytes"]
        except Exception:
            roof["traffic"] = None
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (device-drawn, seeded)",
        "tflops": world * flops_step / (ms_step / 1e3) / 1e12,
        "config": {"workload": WORKLOAD, "layers": L, "batches": MS, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2: consecutive calls read different matrices (96 resident)",
                   "plan": {k: {kk: v[kk] for kk in ("pipeline", "variant", "sm_dec", "grid", "split_k")}
                            for k, v in per.items()}},
        "roofline": roof,
        "per_call": per,
        "footprint": dict(foot, ratio_huffman_form=foot["huffman_form"] / foot["bf16"],
                          ratio_palette_form=foot["palette_form"] / foot["bf16"],
                          per_projection={p: {"ratio_huffman_form": r[1] / r[0], "ratio_palette_form": r[2] / r[0]}
                                          for p, r in per_proj_ratio.items()}),
        "ops_gate_M1": ops,
        "sm_split_down": sm_split,
        "mlp_layer_swiglu": mlp,
        "hard_easy_layers": hard_easy,
        "e2e": {"value": e2e, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "path": "eager uw_gemm calls (ctypes C ABI), UW_PIPE_AUTO"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "setup_s": {"draw_and_compress": t_compress, "autotune": t_tune},
    }
    if rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_profile(args):
    """One call shape, alone, for a profiler's launch list or capture:
    `--profile gate/M=1024` runs that projection's call over the layers of a
    small stack, `--profile step` every projection at every batch of the
    step (the library's own plan choice, no autotuning); `--warmup` passes,
    then `--steps` passes, and it prints the time per pass.  Not a bench
    line."""
    import torch
    import decode_gemm_bf16_b200 as uw
    import synthetic as S

    if args.profile == "step":
        calls = [(p, M) for M in MS for p in PROJ]
    else:
        proj, mpart = args.profile.split("/")
        calls = [(proj, int(mpart.split("=")[1]))]
    used = sorted({PROJ.index(p) for p, _ in calls})
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    blobs = []
    for layer in range(args.layers):
        mats = S.stack_layer_device(layer, dev)
        blobs.append({j: uw.uw_compress(mats[j]) for j in used})
        del mats
    X = {(p, M): S.activations_device(M, SHAPES[p][1], seed=17 + M, device=dev) for p, M in calls}
    Y = {(p, M): torch.empty(M, SHAPES[p][0], dtype=torch.bfloat16, device=dev) for p, M in calls}
    ws = torch.zeros(max(uw.uw_gemm_workspace(blobs[0][PROJ.index(p)], M, args.pipeline) for p, M in calls),
                     dtype=torch.uint8, device=dev)

    def one_pass():
        for p, M in calls:
            j = PROJ.index(p)
            for lb in blobs:
                uw.uw_gemm(X[(p, M)], lb[j], args.pipeline, out=Y[(p, M)], ws=ws, projection=j)

    for _ in range(max(1, args.warmup)):
        one_pass()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        one_pass()
    b.record()
    torch.cuda.synchronize()
    if uw.uw_last_device_status() != 0:
        raise RuntimeError("device status set")
    us = 1e3 * a.elapsed_time(b) / args.steps
    print(json.dumps({"profile": args.profile, "pipeline": args.pipeline, "layers": len(blobs),
                      "calls_per_pass": len(calls) * len(blobs), "us_per_pass": us}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--layers", type=int, default=32, help="layers of the stack (32 = Llama-3.1-8B)")
    ap.add_argument("--stack", action="store_true", help="same as the default run (kept for old command lines)")
    ap.add_argument("--profile", default=None, metavar="PROJ/M=B",
                    help="time one call shape alone (e.g. gate/M=1024) for a profiler; prints no bench line")
    ap.add_argument("--pipeline", default="direct_palette", help="pipeline of the --profile call")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
