"""GPU parity of compression and the three decoders against the CPU oracle.

Every byte of every format section, every decoded stream and every rebuilt
weight must equal the oracle's (integer work: bit-exact).
"""
import numpy as np
import pytest
import torch

import decode_gemm_bf16_b200 as uw
import synthetic as S
from oracle import oracle as O
from tests.gpu_util import dev16, host16, host8, section_view

pytestmark = pytest.mark.gpu


def _constructed():
    N, K = 4, 128
    rng = np.random.default_rng(11)
    ex = rng.integers(110, 126, N * K)
    ex[64 + 17] = 200
    ex[6 * 64 + 63] = 200
    return ((ex.astype(np.uint16) << 7) | rng.integers(0, 128, N * K).astype(np.uint16)).reshape(N, K)


def _high_entropy(N, K):
    """Rows 0-31: sixteen exponents drawn uniformly (4 bits a symbol, more
    stream bits per 8192-weight block than typical weights need); the rest
    Gaussian.  Decoders see both dense and sparse stretches of the stream."""
    rng = np.random.default_rng(12)
    W = S.gaussian_weight(N, K, seed=24)
    ex = rng.integers(112, 128, 32 * K).astype(np.uint16)
    W[:32] = ((ex << 7) | rng.integers(0, 0x8080, 32 * K).astype(np.uint16) & 0x807F).reshape(32, K)
    return W


MATRICES = {
    "small_512x2048": lambda: S.small_matrix()[0],
    "every_pattern_1024x64": S.all_bf16_patterns,
    "constructed_4x128": _constructed,
    "one_exponent_3x128": lambda: (np.full((3, 128), 127, np.uint16) << 7)
    | (np.arange(384, dtype=np.uint16).reshape(3, 128) % 128),
    "tiny_1x64": lambda: (np.array([120] * 32 + [121] * 16 + [122] * 8 + [123] * 8, np.uint16) << 7).reshape(1, 64),
    "nibble_order_1x64": lambda: (np.array([120 + (k % 4) for k in range(64)], np.uint16) << 7).reshape(1, 64),
    "ragged_37x320": lambda: S.gaussian_weight(37, 320, seed=21),
    "ragged_300x1408": lambda: S.weight_with_verbatim_rows(300, 1408, seed=22, frac_groups=0.02),
    "no_verbatim_16x4096": lambda: S.gaussian_weight(16, 4096, seed=23, std=0.5),
    "high_entropy_96x4096": lambda: _high_entropy(96, 4096),
}

_cache = {}


def _pair(name):
    if name not in _cache:
        W = MATRICES[name]()
        _cache[name] = (W, O.compress(W))
    return _cache[name]


def _compare_sections(blob, ob):
    info = blob.info
    assert info["palette"] == ob["palette"].tolist()
    assert info["code_len"] == ob["code_len"].tolist()
    assert info["freq"] == [int(x) for x in ob["freq"]]
    assert info["hist"] == [int(x) for x in ob["hist"]]
    assert info["V"] == ob["V"]
    assert info["total_bits"] == ob["total_bits"]
    assert np.array_equal(section_view(blob, "sm", np.uint8), ob["sm"])
    assert np.array_equal(section_view(blob, "idx", np.uint8), ob["idx"])
    assert np.array_equal(section_view(blob, "vbits", np.uint32), ob["vbits"])
    assert np.array_equal(section_view(blob, "vpre", np.uint32), ob["vpre"])
    assert np.array_equal(section_view(blob, "vexp", np.uint8), ob["vexp"])
    assert np.array_equal(section_view(blob, "vcol", np.uint32), ob["vcol"])
    assert np.array_equal(section_view(blob, "stream", np.uint32), ob["stream"])
    assert np.array_equal(section_view(blob, "chunk_off", np.uint64), ob["chunk_off"])
    assert np.array_equal(section_view(blob, "seg_rel", np.uint16), ob["seg_rel"])


@pytest.mark.parametrize("name", list(MATRICES))
def test_compress_byte_identical(name):
    W, ob = _pair(name)
    blob = uw.uw_compress(dev16(W))
    _compare_sections(blob, ob)
    assert uw.uw_last_device_status() == 0


@pytest.mark.parametrize("name", list(MATRICES))
def test_decoders_match_oracle(name):
    W, ob = _pair(name)
    blob = uw.uw_compress(dev16(W))
    Wd = uw.uw_decode_full(blob)
    E = uw.uw_decode_exponent(blob)
    idx = uw.uw_transcode_palette(blob)
    assert np.array_equal(host16(Wd), W)                     # bit-exact rebuild
    e_oracle, _ = O.split(W)
    assert np.array_equal(host8(E), O.decode_exponent(ob))   # oracle decoder
    assert np.array_equal(host8(E), e_oracle)
    assert np.array_equal(host8(idx), O.transcode(ob))
    assert np.array_equal(host8(idx), ob["idx"])
    assert uw.uw_last_device_status() == 0


def test_index_plane_nibble_order_golden():
    """The library's index plane and transcoder against the hand-derived
    bytes of tests/golden/nibble_order_1x64.txt (0x10, 0x32 repeating:
    element 2j in the low nibble), not only against the oracle."""
    W = MATRICES["nibble_order_1x64"]()
    blob = uw.uw_compress(dev16(W))
    assert section_view(blob, "idx", np.uint8).tolist() == [0x10, 0x32] * 16
    assert host8(uw.uw_transcode_palette(blob)).tolist() == [0x10, 0x32] * 16
    assert [format(int(x), "08X") for x in section_view(blob, "stream", np.uint32)] == \
        ["1B1B1B1B"] * 4 + ["00000000"] * 2
    assert uw.uw_last_device_status() == 0


def test_serialize_matches_oracle_bytes_and_round_trips():
    from tests.test_abi import serialize_oracle
    W, ob = _pair("small_512x2048")
    blob = uw.uw_compress(dev16(W))
    data = uw.uw_blob_serialize(blob)
    assert data == serialize_oracle(ob)
    b2 = uw.uw_blob_deserialize(data)
    assert np.array_equal(host16(uw.uw_decode_full(b2)), W)
    assert np.array_equal(host8(uw.uw_transcode_palette(b2)), ob["idx"])


def test_single_form_blobs():
    W, ob = _pair("ragged_300x1408")
    bh = uw.uw_compress(dev16(W), forms=uw.UW_FORM_HUFFMAN)
    assert bh.info["sections"]["idx"][1] == 0
    assert np.array_equal(host16(uw.uw_decode_full(bh)), W)
    bp = uw.uw_compress(dev16(W), forms=uw.UW_FORM_PALETTE)
    assert bp.info["sections"]["stream"][1] == 0
    assert np.array_equal(section_view(bp, "idx", np.uint8), ob["idx"])
    with pytest.raises(uw.UnweightError) as ei:
        uw.uw_decode_full(bp)
    assert ei.value.status == 4


def test_undecodable_stream_sets_device_status():
    # one exponent -> one symbol with the 1-bit code "0"; a stream of ones has
    # no valid code, which the decoder must report without leaving its buffers
    W, ob = _pair("one_exponent_3x128")
    blob = uw.uw_compress(dev16(W))
    st = blob.section("stream")
    st.fill_(0xFF)
    uw.uw_decode_exponent(blob)
    assert uw.uw_last_device_status() == 8
    assert uw.uw_last_device_status() == 0   # cleared


def test_full_size_gate_projection():
    W = S.gate_projection()
    ob = O.compress(W)
    blob = uw.uw_compress(dev16(W))
    _compare_sections(blob, ob)
    assert np.array_equal(host16(uw.uw_decode_full(blob)), W)
    assert np.array_equal(host8(uw.uw_decode_exponent(blob)), O.split(W)[0])
    assert np.array_equal(host8(uw.uw_transcode_palette(blob)), ob["idx"])
    assert uw.uw_last_device_status() == 0
    info = blob.info
    assert 0.60 < info["bytes_huffman_form"] / (2 * W.size) < 0.72
