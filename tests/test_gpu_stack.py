"""The layer-stack report (bench.py --stack): compression of a Llama-3.1-8B
shaped MLP layer (gate, up, down) kept resident, footprint per form and the
autotuner's plan for batch sizes 1-1024, on one layer."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stack_report_one_layer():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--stack", "--layers", "1"],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    st = line["stack"]
    assert st["matrices"] == 3 and st["weights"] == 3 * 14336 * 4096
    # Huffman form ~0.67 and palette form ~0.76 of BF16 for these weights
    assert 0.6 < st["ratio_huffman_form"] < 0.72 and 0.7 < st["ratio_palette_form"] < 0.8
    plan = line["plan_layer0"]
    assert len(plan) == 3 * 5
    assert {e["M"] for e in plan} == {1, 8, 64, 256, 1024}
    assert all(e["us"] > 0 for e in plan)
