"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point the header declares, and rejects bad shapes and corrupt
serialized blobs on the host before anything would be launched."""
import ctypes
import os
import re
import struct

import numpy as np
import pytest

import decode_gemm_bf16_b200 as uw
from decode_gemm_bf16_b200 import build as uwbuild
from oracle import oracle as O
import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "unweight.h")


@pytest.fixture(scope="module")
def L():
    uwbuild.build()
    return uw.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(uw_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["uw_compress_query", "uw_compress_commit", "uw_decode_full", "uw_decode_exponent",
                 "uw_transcode_palette", "uw_gemm", "uw_autotune", "uw_dense_gemm"]:
        assert must in names


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert sorted(uw.EXPORTS) == declared_functions()


def test_status_strings(L):
    for k, v in uw.STATUS.items():
        assert uw.status_str(k) == v
    assert uw.status_str(99) == "UW_ERR_UNKNOWN"
    assert uw.uw_version() >= 10000


def test_shape_validation_on_host(L):
    n = ctypes.c_size_t()
    assert L.uw_compress_scratch_bytes(512, 2048, ctypes.byref(n)) == 0 and n.value > 0
    assert L.uw_compress_scratch_bytes(512, 100, ctypes.byref(n)) == 2      # K % 64
    assert L.uw_compress_scratch_bytes(512, 0, ctypes.byref(n)) == 2        # empty K
    assert L.uw_compress_scratch_bytes(0, 64, ctypes.byref(n)) == 2         # empty N
    assert L.uw_compress_scratch_bytes(1 << 20, 1 << 12, ctypes.byref(n)) == 2   # > 2^31 elements
    assert L.uw_compress_scratch_bytes((1 << 31) // 4096 - 1, 4096, ctypes.byref(n)) == 0
    assert L.uw_dense_gemm_workspace(4, 512, 2048, 0, 0, 0, ctypes.byref(n)) == 0
    assert L.uw_dense_gemm_workspace(0, 512, 2048, 0, 0, 0, ctypes.byref(n)) == 0 and n.value == 0
    assert L.uw_dense_gemm_workspace(4, 512, 96, 0, 0, 0, ctypes.byref(n)) == 2
    assert L.uw_dense_gemm_workspace(4, 512, 2048, 3, 0, 0, ctypes.byref(n)) == 1       # no such variant
    assert L.uw_dense_gemm_workspace(4, 512, 2048, 0, 0, -1, ctypes.byref(n)) == 1      # negative split
    # one CTA per output tile: no fix-up scratch beyond the minimum
    assert L.uw_dense_gemm_workspace(1024, 14336, 4096, 0, 0, 1, ctypes.byref(n)) == 0 and n.value == 256
    # null pointers are rejected before any device work
    h = ctypes.c_void_p()
    db = ctypes.c_size_t()
    assert L.uw_compress_query(None, 4, 64, 3, None, 0, None, ctypes.byref(h), ctypes.byref(db)) == 1
    assert L.uw_gemm(None, 1, None, None, None, None) == 1
    assert L.uw_decode_full(None, None, None) == 1


# -------- serialized blobs assembled from the oracle's sections -------------
# Header layout of the serialized form (little endian, see the format notes):
#   u32 magic 'UWB1', u32 version 1, i64 N, i64 K, u32 forms, u32 pad,
#   i64 V, i64 nwords, u64 total_bits, u8 palette[16], u8 code_len[16],
#   u64 freq[16], u64 hist[256], u64 bytes[10]; then the nine stored sections.
def serialize_oracle(b, forms=3):
    N, K = b["N"], b["K"]
    secs = [b["sm"].tobytes(), b["vbits"].tobytes(), b["vpre"].tobytes(), b["vexp"].tobytes(),
            b["vcol"].tobytes(),
            b["idx"].tobytes() if forms & 2 else b"",
            b["stream"].tobytes() if forms & 1 else b"",
            b["chunk_off"].tobytes() if forms & 1 else b"",
            b["seg_rel"].tobytes() if forms & 1 else b""]
    lens = [len(s) for s in secs] + [0]
    hdr = struct.pack("<IIqqIIqqQ", 0x31425755, 1, N, K, forms, 0, b["V"],
                      b["stream"].size if forms & 1 else 0, b["total_bits"] if forms & 1 else 0)
    hdr += bytes(b["palette"].tolist()) + bytes(b["code_len"].tolist())
    hdr += struct.pack("<16Q", *[int(x) for x in b["freq"]])
    hdr += struct.pack("<256Q", *[int(x) for x in b["hist"]])
    hdr += struct.pack("<10Q", *lens)
    return hdr + b"".join(secs)


def test_oracle_blob_passes_host_validation(L):
    W, _ = S.small_matrix()
    b = O.compress(W)
    data = serialize_oracle(b)
    assert uw.uw_blob_device_bytes(data) >= len(data) - 700


@pytest.mark.parametrize("what", ["magic", "shape", "codelen", "kraft", "total_bits", "truncate",
                                  "palette_dup", "freq_sum"])
def test_corrupt_headers_rejected(L, what):
    W, _ = S.small_matrix()
    b = O.compress(W)
    if what == "codelen":
        b["code_len"] = b["code_len"].copy()
        b["code_len"][15] = 13
    elif what == "kraft":
        b["code_len"] = b["code_len"].copy()
        b["code_len"][0] += 1
    elif what == "total_bits":
        b["total_bits"] += 1
    elif what == "palette_dup":
        b["palette"] = b["palette"].copy()
        b["palette"][3] = b["palette"][2]
    elif what == "freq_sum":
        b["freq"] = b["freq"].copy()
        b["freq"][0] += 1
    data = bytearray(serialize_oracle(b))
    if what == "magic":
        data[0] ^= 1
    elif what == "shape":
        struct.pack_into("<q", data, 16, 100)   # K = 100
    elif what == "truncate":
        data = data[:-10]
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_blob_device_bytes(bytes(data))
    assert ei.value.status == 3


def test_header_layout_size():
    # the size the library expects: 4+4+8+8+4+4+8+8+8+16+16+128+2048+80
    assert len(serialize_oracle(O.compress(np.zeros((1, 64), np.uint16) | 0x3F80), forms=3)) > 2344


def test_code_hash_ignores_comments_only():
    """Measurements (profiles/traffic.json) are keyed to the code hash: it must
    ignore comments and whitespace but not code, strings or build flags."""
    from decode_gemm_bf16_b200 import build as B
    strip = B._strip_comments
    assert strip("a /* x */ b // y\n c") == strip("a b\n\n   c")
    assert strip('s = "//not a comment"; // gone') == 's = "//not a comment";'
    assert strip("x = '/'; /* multi\nline */ y") == "x = '/'; y"
    assert strip("a + b") != strip("a - b")
    assert len(B.code_hash()) == 64
    assert B.kernel_code_hash("k_decode<full>") == B.code_hash("uw_decode.cu")
    assert B.kernel_code_hash("k_gemm_recon<palette>") != B.kernel_code_hash("k_decode<full>")


# -------- autotuned plans (§自動調優機制): file format and UW_PIPE_AUTO lookup
def _write_plan(path, entries):
    import json
    with open(path, "w") as f:
        json.dump({"plan": entries, "trials": []}, f)


def test_plan_json_round_trip_and_resolve(L, tmp_path):
    entries = [dict(projection=0, M=1, pipeline="direct_palette", variant=2, sm_dec=0, grid=0, split_k=0, us=25.0,
                    layer_us=80.0),
               dict(projection=0, M=64, pipeline="exponent", variant=0, sm_dec=74, grid=0, split_k=0, us=30.0,
                    layer_us=90.0),
               dict(projection=1, M=8, pipeline="transcode", variant=1, sm_dec=0, grid=148, split_k=0, us=40.0,
                    layer_us=90.0),
               dict(projection=1, M=256, pipeline="full", variant=0, sm_dec=0, grid=0, split_k=1, us=50.0,
                    layer_us=100.0)]
    path = str(tmp_path / "plan.json")
    _write_plan(path, entries)
    got = uw.uw_plan_load_json(path)
    assert [(e["projection"], e["M"], e["pipeline"], e["variant"], e["sm_dec"], e["grid"], e["split_k"])
            for e in got] == [(e["projection"], e["M"], e["pipeline"], e["variant"], e["sm_dec"], e["grid"],
                               e["split_k"]) for e in entries]
    plan = uw.Plan(got)
    # exact M; the largest tuned M below; the smallest tuned M when none is below
    assert uw.uw_plan_resolve(plan, 0, 1)["pipeline"] == "direct_palette"
    assert uw.uw_plan_resolve(plan, 0, 1)["variant"] == 2
    r = uw.uw_plan_resolve(plan, 0, 1000)
    assert r["pipeline"] == "exponent" and r["sm_dec"] == 74
    assert uw.uw_plan_resolve(plan, 0, 63)["pipeline"] == "direct_palette"
    assert uw.uw_plan_resolve(plan, 1, 1)["pipeline"] == "transcode"
    assert uw.uw_plan_resolve(plan, 1, 1)["grid"] == 148
    r = uw.uw_plan_resolve(plan, 1, 4096)
    assert r["pipeline"] == "full" and r["split_k"] == 1
    # a projection the plan does not cover
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_plan_resolve(plan, 2, 1)
    assert ei.value.status == 1


def test_plan_resolve_passes_concrete_pipelines_through(L):
    o = uw._opts("transcode", sm_dec=5, grid=7, out_f32=True, variant="tensor", split_k=3, stages=4)
    r = uw.GemmOpts()
    assert L.uw_plan_resolve(ctypes.byref(o), 16, ctypes.byref(r)) == 0
    assert (r.pipeline, r.sm_dec, r.grid, r.out_f32, r.variant, r.split_k, r.stages) == (2, 5, 7, 1, 1, 3, 4)
    # AUTO without a plan
    o = uw._opts("auto")
    assert L.uw_plan_resolve(ctypes.byref(o), 16, ctypes.byref(r)) == 1


def test_plan_json_rejects_bad_files(L, tmp_path):
    bad = tmp_path / "bad.json"
    bad.write_text('{"nothing": []}')
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_plan_load_json(str(bad))
    assert ei.value.status == 3
    bad.write_text('{"plan": [{"projection": 0, "pipeline": "full"}]}')       # no M
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_plan_load_json(str(bad))
    assert ei.value.status == 3
    bad.write_text('{"plan": [{"projection": 0, "M": 4, "pipeline": "huffman"}]}')   # unknown pipeline
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_plan_load_json(str(bad))
    assert ei.value.status == 3
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_plan_load_json(str(tmp_path / "missing.json"))
    assert ei.value.status == 1
