"""The benchmark's workload on a two-layer stack (bench.py --layers 2): the
Llama-3.1-8B-shaped MLP matrices compressed and kept resident, the autotuned
plan consumed through UW_PIPE_AUTO for batch 1-1024, the footprint per form,
and the JSON line's keys."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_two_layer_stack():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--layers", "2", "--steps", "3",
                        "--warmup", "3", "--no-cpu"], capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["steps"] == 3
    fp = line["footprint"]
    assert fp["bf16"] == 2 * 2 * 3 * 14336 * 4096
    # Huffman form ~0.67 and palette form ~0.76 of BF16 for these weights
    assert 0.6 < fp["ratio_huffman_form"] < 0.72 and 0.7 < fp["ratio_palette_form"] < 0.8
    per = line["per_call"]
    assert len(per) == 3 * 5
    assert {k.split("=")[1] for k in per} == {"1", "8", "64", "256", "1024"}
    for v in per.values():
        assert v["us"] > 0 and v["dense_us"] > 0 and 0 < v["roofline_frac"]
    assert line["roofline"]["frac"] > 0 and line["e2e"]["value"] > 0
    assert line["gpu_launches"] >= 3 * 2 * 3 * 5
    assert set(line["ops_gate_M1"]) >= {"decode_full", "decode_exponent", "transcode", "gemm_direct_palette"}
