"""GPU parity of Y = X . W^T through the four pipelines and the dense baseline
against the CPU oracle's fp32-accumulated (and fp64) reference.

Tolerance (see tests/gpu_util.py): max relative error 2e-3 element-wise with a
1e-2*rms floor on float32 outputs, plus 2^-8 relative BF16 output rounding on
BF16 outputs.  The rebuilt weights are bit-exact, so pipelines that share the
tiling and split must also agree bit for bit.
"""
import numpy as np
import pytest
import torch

import decode_gemm_bf16_b200 as uw
import synthetic as S
from oracle import oracle as O
from tests.gpu_util import check_gemm, dev16, host16, oracle_gemm

pytestmark = pytest.mark.gpu

PIPES = ["full", "exponent", "transcode", "direct_palette"]

SHAPES = {
    # N x K: several 128-row tiles and 64-wide k steps, ragged N, verbatim rows
    "384x512": lambda: S.weight_with_verbatim_rows(384, 512, seed=31, frac_groups=0.01),
    "200x1408": lambda: S.weight_with_verbatim_rows(200, 1408, seed=32, frac_groups=0.01),
    # K an odd multiple of 64: small batches fall back to 64-k stages
    "136x576": lambda: S.weight_with_verbatim_rows(136, 576, seed=33, frac_groups=0.01),
}
MS = [1, 3, 16, 17, 64, 100, 256, 300]

_cache = {}


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _case(shape):
    if shape not in _cache:
        W = SHAPES[shape]()
        blob = uw.uw_compress(dev16(W))
        _cache[shape] = (W, blob)
    return _cache[shape]


def _f32(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("M", MS)
def test_pipelines_match_oracle(shape, M):
    W, blob = _case(shape)
    X = S.activations(M, W.shape[1], seed=1000 + M)
    R32 = O.gemm(X, W, "f32")
    R64 = O.gemm(X, W, "f64")
    Xd = dev16(X)
    outs = {}
    for pipe in PIPES:
        Y32 = uw.uw_gemm(Xd, blob, pipe, out_f32=True)
        Yb = uw.uw_gemm(Xd, blob, pipe, out_f32=False)
        torch.cuda.synchronize()
        check_gemm(_f32(Y32), R32, bf16_out=False)
        check_gemm(_f32(Y32), R64, bf16_out=False)
        check_gemm(_f32(Yb), R32, bf16_out=True)
        outs[pipe] = (_f32(Y32), host16(Yb))
    Yd = _f32(uw.uw_dense_gemm(Xd, dev16(W), out_f32=True))
    check_gemm(Yd, R32, bf16_out=False)
    for pipe in PIPES:
        assert np.array_equal(outs[pipe][0], Yd), pipe        # same tiles, same split
        assert np.array_equal(outs[pipe][1], outs["full"][1]), pipe
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("grid", [1, 2, 7, 33, 500])
def test_stream_k_splits(grid):
    """Different CTA counts cut the k loop differently; all must match."""
    W, blob = _case("384x512")
    X = S.activations(40, 512, seed=77)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    for pipe in ["exponent", "direct_palette"]:
        Y = uw.uw_gemm(Xd, blob, pipe, out_f32=True, grid=grid)
        check_gemm(_f32(Y), R, bf16_out=False)
    Yd = uw.uw_dense_gemm(Xd, dev16(W), out_f32=True, grid=grid)
    check_gemm(_f32(Yd), R, bf16_out=False)
    assert uw.uw_last_device_status() == 0


def test_repeated_calls_reuse_workspace():
    W, blob = _case("200x1408")
    X = S.activations(17, 1408, seed=5)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    first = None
    for _ in range(4):
        Y = _f32(uw.uw_gemm(Xd, blob, "transcode", out_f32=True, grid=13))
        check_gemm(Y, R, bf16_out=False)
        if first is None:
            first = Y
        assert np.array_equal(Y, first)


def test_empty_batch_and_errors():
    W, blob = _case("384x512")
    Y = torch.empty(0, 384, dtype=torch.bfloat16, device="cuda")
    out = uw.uw_gemm(torch.empty(0, 512, dtype=torch.bfloat16, device="cuda"), blob, "exponent", out=Y)
    assert out.shape == (0, 384)
    bh = uw.uw_compress(dev16(W), forms=uw.UW_FORM_HUFFMAN)
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm(dev16(S.activations(2, 512, 1)), bh, "direct_palette")
    assert ei.value.status == 4
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm(dev16(S.activations(2, 512, 1)), blob, "full", ws=small)
    assert ei.value.status == 5


def _sampled(X, W, Y, n_samples, seed, bf16_out):
    rng = np.random.default_rng(seed)
    M, N = Y.shape
    ms = rng.integers(0, M, n_samples)
    ns = rng.integers(0, N, n_samples)
    ref = np.array([O.gemm_one(X, W, int(m), int(n), "f32") for m, n in zip(ms, ns)])
    # floor from the sampled references' scale
    check_gemm(Y[ms, ns], ref, bf16_out=bf16_out, K=W.shape[1])


@pytest.fixture(scope="module")
def gate_case():
    W = S.gate_projection()
    return W, uw.uw_compress(dev16(W))


@pytest.fixture(scope="module")
def down_case():
    W = S.down_projection()
    return W, uw.uw_compress(dev16(W))


def _full_size_all_paths(W, blob, M, seed):
    """Every output of the four pipelines and the dense baseline, BF16 and
    float32 outputs, against the oracle's fp32-accumulated product."""
    X = S.activations(M, W.shape[1], seed=seed)
    R = oracle_gemm(X, W, "f32")
    K = W.shape[1]
    Xd = dev16(X)
    ref = None
    for pipe in PIPES:
        Yb = _f32(uw.uw_gemm(Xd, blob, pipe))
        check_gemm(Yb, R, bf16_out=True, K=K)
        if ref is None:
            ref = Yb
        assert np.array_equal(Yb, ref), pipe
    check_gemm(_f32(uw.uw_gemm(Xd, blob, "direct_palette", out_f32=True)), R, bf16_out=False, K=K)
    Wd = dev16(W)
    Yd = _f32(uw.uw_dense_gemm(Xd, Wd))
    check_gemm(Yd, R, bf16_out=True, K=K)
    assert np.array_equal(Yd, ref)
    check_gemm(_f32(uw.uw_dense_gemm(Xd, Wd, out_f32=True)), R, bf16_out=False, K=K)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("M", [1, 64, 1024])
def test_full_size_gate_every_output(gate_case, M):
    """Gate projection W[14336,4096] at batch 1 (tensor cores, stream-K over
    the 112 row tiles), 64 (one CTA per tile) and 1024 (stream-K over 448
    tiles): every output element of every path against the oracle."""
    W, blob = gate_case
    _full_size_all_paths(W, blob, M, seed=1 + S.X_SEED_OFFSET + M)


@pytest.mark.parametrize("M", [256, 1024])
def test_full_size_down_every_output(down_case, M):
    """Down projection W[4096,14336] (32 row tiles, K = 14336) at batch 256
    (four CTAs per tile) and 1024 (one CTA per tile, 128 tiles)."""
    W, blob = down_case
    _full_size_all_paths(W, blob, M, seed=4 + S.X_SEED_OFFSET + M)


@pytest.mark.parametrize("M", [1, 16])
def test_full_size_down_small_batch(down_case, M):
    """Down projection at batch 1 (the CUDA-core GEMV serves it) and 16
    (tensor cores, 128-k stages, each tile cut ~4-5 ways): every output."""
    W, blob = down_case
    _full_size_all_paths(W, blob, M, seed=40 + M)


@pytest.mark.parametrize("fill", [0x00, 0xFF, "random"])
def test_workspace_contents_do_not_matter(fill):
    """Fix-up counters carry a per-call tag, so stale bytes left in the
    workspace by other calls (other pipelines, other layouts) are harmless."""
    W, blob = _case("384x512")
    X = S.activations(33, 512, seed=9)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    need = max(uw.uw_gemm_workspace(blob, 33, p) for p in PIPES)
    ws = torch.empty(need + 4096, dtype=torch.uint8, device="cuda")
    for pipe in PIPES + ["dense"]:
        if fill == "random":
            ws.random_(0, 256)
        else:
            ws.fill_(fill)
        if pipe == "dense":
            Y = uw.uw_dense_gemm(Xd, dev16(W), out_f32=True, ws=ws)
        else:
            Y = uw.uw_gemm(Xd, blob, pipe, out_f32=True, ws=ws)
        check_gemm(_f32(Y), R, bf16_out=False)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("pipe", ["full", "exponent", "transcode"])
@pytest.mark.parametrize("sm_dec", [1, 37, 148, 300])
def test_decoder_beside_gemm(pipe, sm_dec):
    """Decoder CTAs running beside the GEMM (SM split): the GEMM waits for
    each 128-row band; the result is the same as decode-then-GEMM with one
    k range per CTA (the split the GEMM beside a decoder uses)."""
    W, blob = _case("200x1408")
    X = S.activations(24, 1408, seed=11)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    ref = _f32(uw.uw_gemm(Xd, blob, pipe, out_f32=True, grid=_sms()))
    for _ in range(2):
        Y = _f32(uw.uw_gemm(Xd, blob, pipe, out_f32=True, sm_dec=sm_dec))
        check_gemm(Y, R, bf16_out=False)
        assert np.array_equal(Y, ref)
    assert uw.uw_last_device_status() == 0


def test_decoder_beside_gemm_full_size(gate_case):
    W, blob = gate_case
    X = S.activations(16, 4096, seed=12)
    Xd = dev16(X)
    for pipe in ["exponent", "transcode"]:
        ref = _f32(uw.uw_gemm(Xd, blob, pipe, grid=_sms()))   # one k range per CTA, as beside a decoder
        Y = _f32(uw.uw_gemm(Xd, blob, pipe, sm_dec=74))
        assert np.array_equal(Y, ref)
        _sampled(X, W, Y, 64, seed=5, bf16_out=True)
    assert uw.uw_last_device_status() == 0


def test_autotune_plan(tmp_path):
    """The autotuner (§自動調優機制) over two copies of a three-projection
    layer: one entry per projection and batch, each the measured minimum of
    its candidates in the last round of the descent (within the 1% it
    requires before it moves), the plan file reads back, and UW_PIPE_AUTO
    under the plan matches the oracle."""
    import json
    shapes = [(384, 512), (384, 512), (512, 384 + 128)]
    Ws = [S.gaussian_weight(n, k, seed=60 + i) for i, (n, k) in enumerate(shapes)]
    copies = 2
    blobs = [uw.uw_compress(dev16(w)) for _ in range(copies) for w in Ws]
    Ms = [1, 64]
    Xh = [S.activations(max(Ms), k, seed=70 + i) for i, (n, k) in enumerate(shapes)]
    Xs = [dev16(x) for x in Xh]
    Ys = [torch.empty(max(Ms), n, dtype=torch.bfloat16, device="cuda") for (n, k) in shapes]
    need = max(uw.uw_gemm_workspace(b, max(Ms), p, sm_dec=sd) for b in blobs[:3]
               for p in PIPES for sd in (0, 300))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    path = str(tmp_path / "plan.json")
    plan = uw.uw_autotune(blobs, Ms, Xs, Ys, ws, reps=3, plan_json_path=path, copies=copies)
    assert len(plan) == len(Ms) * len(shapes)
    for i, e in enumerate(plan):
        assert e["M"] == Ms[i // 3] and e["projection"] == i % 3
        assert e["pipeline"] in PIPES and e["us"] > 0 and e["layer_us"] > 0
    saved = json.load(open(path))
    assert [(d["projection"], d["M"], d["pipeline"], d["variant"], d["sm_dec"], d["grid"], d["split_k"])
            for d in saved["plan"]] == [(e["projection"], e["M"], e["pipeline"], e["variant"], e["sm_dec"],
                                         e["grid"], e["split_k"]) for e in plan]
    trials = saved["trials"]
    for M in Ms:
        last = max(t["round"] for t in trials if t["M"] == M)
        chosen = {e["projection"]: e for e in plan if e["M"] == M}
        for proj in range(3):
            ts = [t for t in trials if t["M"] == M and t["round"] == last and t["projection"] == proj
                  and t["layer_us"] > 0]
            # no candidate of the last round beat the chosen configuration by 1%
            assert all(t["layer_us"] >= 0.99 * chosen[proj]["layer_us"] for t in ts), (M, proj)
            assert len(ts) >= 1
    # the plan file is the per-model configuration: read it back and run AUTO
    loaded = uw.uw_plan_load_json(path)
    assert [(e["projection"], e["M"], e["pipeline"]) for e in loaded] == \
        [(e["projection"], e["M"], e["pipeline"]) for e in plan]
    P = uw.Plan(loaded)
    for M in [1, 5, 64, 100]:
        for proj, (n, k) in enumerate(shapes):
            X = Xh[proj][:M]
            Y = uw.uw_gemm(dev16(X), blobs[proj], "auto", plan=P, projection=proj)
            check_gemm(_f32(Y), O.gemm(X, Ws[proj], "f32"), bf16_out=True)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("variant", ["tensor", "gemv"])
def test_variant_forced_at_batch_one(variant):
    """Batch 1 forced onto the tensor cores or onto the CUDA-core GEMV: each
    matches the oracle, and all pipelines agree bit for bit within a variant."""
    W, blob = _case("384x512")
    X = S.activations(1, 512, seed=91)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    ref = None
    for pipe in PIPES:
        Y = _f32(uw.uw_gemm(Xd, blob, pipe, out_f32=True, variant=variant))
        check_gemm(Y, R, bf16_out=False)
        if ref is None:
            ref = Y
        assert np.array_equal(Y, ref), pipe
    assert np.array_equal(_f32(uw.uw_dense_gemm(Xd, dev16(W), out_f32=True, variant=variant)), ref)
    # the GEMV serves batch 1 only
    if variant == "gemv":
        with pytest.raises(uw.UnweightError) as ei:
            uw.uw_gemm(dev16(S.activations(2, 512, seed=92)), blob, "direct_palette", variant="gemv")
        assert ei.value.status == 4
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("split_k", [1, 2, 3, 8])
@pytest.mark.parametrize("M", [5, 64, 200])
def test_split_k_and_stages(split_k, M):
    """Every output tile cut into split_k k ranges (one CTA each), with the
    ring held to two stages: matches the oracle, pipelines agree."""
    W, blob = _case("200x1408")
    X = S.activations(M, 1408, seed=93 + M)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    ref = None
    for pipe in PIPES:
        for stages in (0, 2):
            Y = _f32(uw.uw_gemm(Xd, blob, pipe, out_f32=True, split_k=split_k, stages=stages))
            check_gemm(Y, R, bf16_out=False)
            if ref is None:
                ref = Y
            assert np.array_equal(Y, ref), (pipe, stages)
    assert uw.uw_last_device_status() == 0


def test_default_grid_uneven_k_ranges():
    """The default grid with 64-row batch tiles and fewer tiles than SMs cuts
    every tile into floor(SMs / tiles) k ranges: N = 1024 gives 8 tiles, so
    18 ranges over 32 k steps of 128 (uneven).  Every output against the
    oracle, and bit for bit against the dense baseline."""
    W = S.weight_with_verbatim_rows(1024, 4096, seed=94, frac_groups=0.01)
    blob = uw.uw_compress(dev16(W))
    X = S.activations(64, 4096, seed=95)
    R = oracle_gemm(X, W, "f32")
    Xd = dev16(X)
    Yd = _f32(uw.uw_dense_gemm(Xd, dev16(W), out_f32=True))
    check_gemm(Yd, R, bf16_out=False)
    for pipe in PIPES:
        Y = _f32(uw.uw_gemm(Xd, blob, pipe, out_f32=True))
        check_gemm(Y, R, bf16_out=False)
        assert np.array_equal(Y, Yd), pipe
    assert uw.uw_last_device_status() == 0


_TIMEOUT_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import decode_gemm_bf16_b200 as uw, synthetic as S
from tests.gpu_util import dev16
from oracle import oracle as O
W = S.weight_with_verbatim_rows(200, 1408, seed=32, frac_groups=0.01)
blob = uw.uw_compress(dev16(W))
X = S.activations(24, 1408, seed=11)
Xd = dev16(X)
# decoder beside the GEMM, but no decoder launched: the GEMM's bounded waits
# for its bands run out and report UW_ERR_TIMEOUT
uw.uw_gemm(Xd, blob, "transcode", sm_dec=37)
print("status", uw.uw_last_device_status())
# the context stays usable: a normal call afterwards is correct
Y = uw.uw_gemm(Xd, blob, "transcode", out_f32=True).double().cpu().numpy()
R = O.gemm(X, W, "f32")
print("after", uw.uw_last_device_status(), float(np.abs(Y - R).max() / np.abs(R).max()))
"""


def test_bounded_wait_expires_with_timeout_status():
    """A device-side wait that nothing satisfies (a decoder band never
    published, via the UW_DEBUG_SKIP_DECODER hook) ends after UW_TIMEOUT_MS
    with UW_ERR_TIMEOUT in the device status word; the process keeps using
    the GPU normally afterwards.  Runs in a child process so the short
    timeout and the hook stay out of the other tests."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, UW_TIMEOUT_MS="20", UW_DEBUG_SKIP_DECODER="1")
    r = subprocess.run([sys.executable, "-c", _TIMEOUT_CHILD, root], env=env, capture_output=True, text=True,
                       timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = dict(l.split(" ", 1) for l in r.stdout.strip().splitlines() if " " in l)
    assert int(lines["status"]) == 7          # UW_ERR_TIMEOUT
    after = lines["after"].split()
    assert int(after[0]) == 0 and float(after[1]) < 1e-2


# ---------------------------------------------------------------------------
# Fused Huffman-decode product (UW_PIPE_FUSED_HUFFMAN): the stream is decoded
# inside the product, no decoded plane goes to HBM.
# ---------------------------------------------------------------------------
FUSED_SHAPES = {
    "384x512": lambda: S.weight_with_verbatim_rows(384, 512, seed=31, frac_groups=0.01),
    "200x1024": lambda: S.weight_with_verbatim_rows(200, 1024, seed=34, frac_groups=0.02),
    "high_entropy_96x4096": lambda: _high_entropy_rows(96, 4096),
}


def _high_entropy_rows(N, K):
    rng = np.random.default_rng(12)
    W = S.gaussian_weight(N, K, seed=24)
    ex = rng.integers(112, 128, 32 * K).astype(np.uint16)
    W[:32] = ((ex << 7) | rng.integers(0, 0x8080, 32 * K).astype(np.uint16) & 0x807F).reshape(32, K)
    return W


_fcache = {}


def _fcase(shape):
    if shape not in _fcache:
        W = FUSED_SHAPES[shape]()
        _fcache[shape] = (W, uw.uw_compress(dev16(W)))
    return _fcache[shape]


@pytest.mark.parametrize("shape", list(FUSED_SHAPES))
@pytest.mark.parametrize("M", [1, 2, 3, 8, 16, 17, 40])
def test_fused_huffman_matches_oracle(shape, M):
    W, blob = _fcase(shape)
    X = S.activations(M, W.shape[1], seed=2000 + M)
    R32 = O.gemm(X, W, "f32")
    Xd = dev16(X)
    Y32 = _f32(uw.uw_gemm(Xd, blob, "fused_huffman", out_f32=True))
    check_gemm(Y32, R32, bf16_out=False)
    check_gemm(Y32, O.gemm(X, W, "f64"), bf16_out=False)
    Yb = _f32(uw.uw_gemm(Xd, blob, "fused_huffman"))
    check_gemm(Yb, R32, bf16_out=True)
    # deterministic: the same call gives the same bits
    assert np.array_equal(_f32(uw.uw_gemm(Xd, blob, "fused_huffman", out_f32=True)), Y32)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("M", [1, 4])
def test_fused_huffman_graph_replays(M):
    """Captured once and replayed: the per-call tag is reused, so the last
    warp of each row group resets its counter; every replay must match
    (batch 1: one CTA per SM with staged stream words; batch 4: 8-warp CTAs)."""
    W, blob = _fcase("200x1024")
    X = S.activations(M, 1024, seed=2100)
    R = O.gemm(X, W, "f32")
    Xd = dev16(X)
    Y = torch.empty(M, 200, dtype=torch.float32, device="cuda")
    ws = torch.zeros(uw.uw_gemm_workspace(blob, M, "fused_huffman"), dtype=torch.uint8, device="cuda")
    uw.uw_gemm(Xd, blob, "fused_huffman", out=Y, out_f32=True, ws=ws)
    torch.cuda.synchronize()
    first = _f32(Y)
    check_gemm(first, R, bf16_out=False)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        uw.uw_gemm(Xd, blob, "fused_huffman", out=Y, out_f32=True, ws=ws)
    for _ in range(3):
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(_f32(Y), first)
    assert uw.uw_last_device_status() == 0


def test_fused_huffman_rejects_unsupported():
    W, blob = _case("200x1408")            # K = 1408 is not a multiple of 256
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm(dev16(S.activations(2, 1408, 1)), blob, "fused_huffman")
    assert ei.value.status == 4
    Wp, _ = _fcase("384x512")
    bp = uw.uw_compress(dev16(Wp), forms=uw.UW_FORM_PALETTE)   # no Huffman form
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm(dev16(S.activations(2, 512, 1)), bp, "fused_huffman")
    assert ei.value.status == 4


@pytest.mark.parametrize("M", [1, 2, 16, 64])
def test_fused_huffman_full_size_gate(gate_case, M):
    W, blob = gate_case
    X = S.activations(M, 4096, seed=2200 + M)
    R = oracle_gemm(X, W, "f32")
    check_gemm(_f32(uw.uw_gemm(dev16(X), blob, "fused_huffman")), R, bf16_out=True)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("M", [1, 16, 64])
def test_fused_huffman_full_size_down(down_case, M):
    W, blob = down_case
    X = S.activations(M, 14336, seed=2300 + M)
    R = oracle_gemm(X, W, "f32")
    check_gemm(_f32(uw.uw_gemm(dev16(X), blob, "fused_huffman")), R, bf16_out=True, K=14336)
    assert uw.uw_last_device_status() == 0


# ---------------------------------------------------------------------------
# Gate + up in one launch with the SwiGLU epilogue (uw_gemm_swiglu)
# ---------------------------------------------------------------------------
SWIGLU_PAIRS = {
    "384x512": lambda: (S.weight_with_verbatim_rows(384, 512, seed=51, frac_groups=0.01),
                        S.weight_with_verbatim_rows(384, 512, seed=52, frac_groups=0.01)),
    "200x1408": lambda: (S.weight_with_verbatim_rows(200, 1408, seed=53, frac_groups=0.01),
                         S.gaussian_weight(200, 1408, seed=54, std=0.03)),
}
_scache = {}


def _scase(name):
    if name not in _scache:
        Wg, Wu = SWIGLU_PAIRS[name]()
        _scache[name] = (Wg, Wu, uw.uw_compress(dev16(Wg)), uw.uw_compress(dev16(Wu)))
    return _scache[name]


@pytest.mark.parametrize("name", list(SWIGLU_PAIRS))
@pytest.mark.parametrize("M", [1, 3, 16, 17, 64, 100, 128, 129, 300])
def test_swiglu_matches_oracle(name, M):
    from tests.gpu_util import check_swiglu
    Wg, Wu, bg, bu = _scase(name)
    X = S.activations(M, Wg.shape[1], seed=3000 + M)
    G = O.gemm(X, Wg, "f32")
    U = O.gemm(X, Wu, "f32")
    Xd = dev16(X)
    H32 = _f32(uw.uw_gemm_swiglu(Xd, bg, bu, out_f32=True))
    check_swiglu(H32, G, U, bf16_out=False)
    Hb = _f32(uw.uw_gemm_swiglu(Xd, bg, bu))
    check_swiglu(Hb, G, U, bf16_out=True)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("opts", [dict(grid=7), dict(grid=1), dict(split_k=1), dict(split_k=3), dict(stages=2),
                                  dict(variant="tensor")])
def test_swiglu_splits(opts):
    """Stream-K and whole-multiple splits cut the paired accumulators; the
    finisher adds both halves before the SwiGLU.  All splits agree with the
    oracle."""
    from tests.gpu_util import check_swiglu
    Wg, Wu, bg, bu = _scase("384x512")
    for M in (5, 80, 200):
        X = S.activations(M, 512, seed=3100 + M)
        H = _f32(uw.uw_gemm_swiglu(dev16(X), bg, bu, out_f32=True, **opts))
        check_swiglu(H, O.gemm(X, Wg, "f32"), O.gemm(X, Wu, "f32"), bf16_out=False)
    assert uw.uw_last_device_status() == 0


def test_swiglu_rejects_unsupported():
    Wg, Wu, bg, bu = _scase("384x512")
    X = dev16(S.activations(2, 512, seed=1))
    for kw in (dict(pipeline="exponent"), dict(variant="gemv")):
        with pytest.raises(uw.UnweightError) as ei:
            uw.uw_gemm_swiglu(X, bg, bu, **kw)
        assert ei.value.status == 4
    _, _, b2, _ = _scase("200x1408")
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm_swiglu(X, bg, b2)
    assert ei.value.status == 2
    bh = uw.uw_compress(dev16(Wu), forms=uw.UW_FORM_HUFFMAN)
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm_swiglu(X, bg, bh)
    assert ei.value.status == 4


@pytest.fixture(scope="module")
def gate_up_case():
    Wg = S.gate_projection(seed=2)
    Wu = S.gate_projection(seed=3)
    return Wg, Wu, uw.uw_compress(dev16(Wg)), uw.uw_compress(dev16(Wu))


@pytest.mark.parametrize("M", [1, 64, 256])
def test_swiglu_full_size_every_output(gate_up_case, M):
    """The Llama-3.1-8B gate+up pair W[14336,4096] x 2: every element of H
    against the oracle."""
    from tests.gpu_util import check_swiglu
    Wg, Wu, bg, bu = gate_up_case
    X = S.activations(M, 4096, seed=2 + S.X_SEED_OFFSET + M)
    G = oracle_gemm(X, Wg, "f32")
    U = oracle_gemm(X, Wu, "f32")
    check_swiglu(_f32(uw.uw_gemm_swiglu(dev16(X), bg, bu)), G, U, bf16_out=True)
    assert uw.uw_last_device_status() == 0


def test_swiglu_full_size_large_batch_sampled(gate_up_case):
    """M = 1024 (eight 128-row batch tiles): sampled outputs against the
    oracle, one output element at a time."""
    Wg, Wu, bg, bu = gate_up_case
    M = 1024
    X = S.activations(M, 4096, seed=2 + S.X_SEED_OFFSET + M)
    H = _f32(uw.uw_gemm_swiglu(dev16(X), bg, bu))
    rng = np.random.default_rng(9)
    ms, ns = rng.integers(0, M, 512), rng.integers(0, 14336, 512)
    G = np.array([O.gemm_one(X, Wg, int(m), int(n), "f32") for m, n in zip(ms, ns)])
    U = np.array([O.gemm_one(X, Wu, int(m), int(n), "f32") for m, n in zip(ms, ns)])
    from tests.gpu_util import check_swiglu
    check_swiglu(H[ms, ns], G, U, bf16_out=True)
    assert uw.uw_last_device_status() == 0


# ---------------------------------------------------------------------------
# Layer sequences with hard (Huffman, transcoded ahead) and easy (palette)
# projections (uw_gemm_sequence)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("pattern", ["hehe", "hhhh", "eeee", "ehhe"])
@pytest.mark.parametrize("dec_ctas", [0, 37])
@pytest.mark.parametrize("M", [1, 16, 100])
def test_sequence_chain_matches_oracle(pattern, dec_ctas, M):
    """A chain of four 512x512 projections, item i reading item i-1's BF16
    output.  Each item's output against the oracle on the input the GPU fed
    it, and bit for bit against the same item run alone."""
    n = len(pattern)
    Ws = [S.weight_with_verbatim_rows(512, 512, seed=400 + i, frac_groups=0.01) for i in range(n)]
    blobs = [uw.uw_compress(dev16(w)) for w in Ws]
    X0 = dev16(S.activations(M, 512, seed=410 + M))
    Ys = [torch.empty(M, 512, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    items = [(blobs[i], X0 if i == 0 else Ys[i - 1], Ys[i], pattern[i] == "h") for i in range(n)]
    for rep in range(2):
        for y in Ys:
            y.fill_(float("nan"))
        uw.uw_gemm_sequence(items, M, dec_ctas=dec_ctas)
        torch.cuda.synchronize()
        xin = X0
        for i in range(n):
            Xh = host16(xin)
            check_gemm(_f32(Ys[i]), O.gemm(Xh, Ws[i], "f32"), bf16_out=True)
            alone = uw.uw_gemm(xin, blobs[i], "transcode" if pattern[i] == "h" else "direct_palette", variant="tensor")
            assert np.array_equal(host16(alone), host16(Ys[i])), (i, rep)
            xin = Ys[i]
    assert uw.uw_last_device_status() == 0


def test_sequence_rejects_missing_forms():
    W = S.gaussian_weight(256, 512, seed=420)
    bp = uw.uw_compress(dev16(W), forms=uw.UW_FORM_PALETTE)
    X = dev16(S.activations(4, 512, seed=1))
    Y = torch.empty(4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_gemm_sequence([(bp, X, Y, True)], 4)
    assert ei.value.status == 4


@pytest.mark.parametrize("M", [1, 16])
def test_repeated_calls_bit_identical_full_size(gate_up_case, M):
    """The same call thirty times in a row gives the same bits (the split and
    the summation order depend on the shape only).  Out-of-order completions
    of the stage ring's loads once let a rebuild group run ahead into a slot
    whose tiles had not landed (an odd ring); repeats catch that kind of race."""
    Wg, Wu, bg, bu = gate_up_case
    X = dev16(S.activations(M, 4096, seed=4000 + M))
    calls = {"swiglu": lambda: uw.uw_gemm_swiglu(X, bg, bu, out_f32=True),
             "direct_palette": lambda: uw.uw_gemm(X, bg, "direct_palette", out_f32=True),
             "exponent": lambda: uw.uw_gemm(X, bu, "exponent", out_f32=True)}
    for name, fn in calls.items():
        ref = fn().clone()
        for _ in range(30):
            assert torch.equal(fn(), ref), name
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("M", [1, 5, 16])
def test_small_batch_full_size_gate_repeats(gate_case, M):
    """Batch tiles of 16 rows on the default grid (stream-K over one CTA per
    SM, cut tiles finished from the partials of the others): every output
    against the oracle; repeated calls, and a CUDA graph replaying four of
    them on one workspace (the per-row tags of one call must not be taken
    for the next call's), give the same bits."""
    W, blob = gate_case
    X = S.activations(M, 4096, seed=120 + M)
    Xd = dev16(X)
    R = oracle_gemm(X, W, "f32")
    Y = _f32(uw.uw_gemm(Xd, blob, "direct_palette", out_f32=True))
    check_gemm(Y, R, bf16_out=False)
    for _ in range(3):
        assert np.array_equal(_f32(uw.uw_gemm(Xd, blob, "direct_palette", out_f32=True)), Y)
    assert np.array_equal(_f32(uw.uw_gemm(Xd, blob, "direct_palette", out_f32=True, grid=_sms())), Y)
    outs = [torch.empty(M, W.shape[0], dtype=torch.float32, device="cuda") for _ in range(4)]
    ws = torch.zeros(uw.uw_gemm_workspace(blob, M, "direct_palette"), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for o in outs:
            uw.uw_gemm(Xd, blob, "direct_palette", out=o, out_f32=True, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for o in outs:
            uw.uw_gemm(Xd, blob, "direct_palette", out=o, out_f32=True, ws=ws)
    for _ in range(3):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for o in outs:
            assert np.array_equal(o.cpu().numpy(), Y)
    del g
    assert uw.uw_last_device_status() == 0


def test_dense_agrees_with_palette_batch8():
    """The dense baseline and the rebuilding pipelines share the tile and
    k-range split: equal bits at batch 8 on 40 row tiles cut by stream-K."""
    W = S.weight_with_verbatim_rows(5120, 2048, seed=130, frac_groups=0.01)
    blob = uw.uw_compress(dev16(W))
    X = S.activations(8, 2048, seed=131)
    Xd = dev16(X)
    R = O.gemm(X, W, "f32")
    Yd = _f32(uw.uw_dense_gemm(Xd, dev16(W), out_f32=True))
    check_gemm(Yd, R, bf16_out=False)
    for pipe in ["exponent", "transcode", "direct_palette"]:
        assert np.array_equal(_f32(uw.uw_gemm(Xd, blob, pipe, out_f32=True)), Yd), pipe
    assert uw.uw_last_device_status() == 0
