"""Pins for the CPU oracle (no GPU).

The oracle is only trusted once it agrees with facts that do not come from
itself: IEEE/BF16 field positions, hand-derived tiny streams, textbook Huffman
examples (CLRS section 16.3, RFC 1951 section 3.2.2), brute-force enumeration
of length vectors, closed-form Gaussian exponent statistics, exact rational
arithmetic for tiny products, and the figures printed on the Unweight page
("Cloudflare推出Unweight無損壓縮系統", §BF16權重壓縮原理: top-16 exponents cover
>99% of weights, ~2.6 bits of information).
"""
import itertools
import heapq
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import synthetic as S
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# --------------------------------------------------------------------------
# split / merge: BF16 = sign(1) | exponent(8) | mantissa(7)
# --------------------------------------------------------------------------
def test_split_known_patterns():
    # IEEE-754 binary16-brain facts: 1.0 = 0x3F80, -2.0 = 0xC000,
    # smallest subnormal 0x0001, +inf 0x7F80, a quiet NaN 0x7FC1, -0 = 0x8000.
    w = np.array([0x3F80, 0xC000, 0x0001, 0x7F80, 0x7FC1, 0x8000, 0x3F81], np.uint16)
    e, sm = O.split(w)
    assert list(e) == [127, 128, 0, 255, 255, 0, 127]
    assert list(sm) == [0x00, 0x80, 0x01, 0x00, 0x41, 0x80, 0x01]


def test_split_merge_bijection_all_patterns():
    w = S.all_bf16_patterns().reshape(-1)
    e, sm = O.split(w)
    assert np.array_equal(O.merge(e, sm), w)
    # every (e, sm) pair appears exactly once
    pairs = e.astype(np.int64) * 256 + sm
    assert np.unique(pairs).size == 65536


# --------------------------------------------------------------------------
# histogram / palette
# --------------------------------------------------------------------------
def _pow2_bits(expo):
    """BF16 bit pattern of 2**(expo-127) (positive, mantissa 0)."""
    return np.uint16(int(expo) << 7)


def test_histogram_constructed():
    rng = np.random.default_rng(5)
    counts = {3: 7, 100: 1, 127: 40, 200: 13, 255: 2}
    vals = np.concatenate([np.full(c, _pow2_bits(e), np.uint16) for e, c in counts.items()])
    # random signs and mantissas must not change the exponent
    vals = vals | (rng.integers(0, 2, vals.size).astype(np.uint16) << 15) | rng.integers(0, 128, vals.size).astype(np.uint16)
    rng.shuffle(vals)
    e, _ = O.split(vals)
    h = O.histogram(e)
    expect = np.zeros(256, np.uint64)
    for k, c in counts.items():
        expect[k] = c
    assert np.array_equal(h, expect)


def test_palette_ranking_and_padding():
    h = np.zeros(256, np.uint64)
    h[5] = 10
    h[3] = 10
    h[200] = 50
    h[7] = 1
    pal, inv = O.palette(h)
    # count desc, exponent asc on ties; then the smallest absent exponents
    assert list(pal) == [200, 3, 5, 7, 0, 1, 2, 4, 6, 8, 9, 10, 11, 12, 13, 14]
    assert inv[200] == 0 and inv[3] == 1 and inv[5] == 2 and inv[7] == 3 and inv[14] == 15
    assert inv[15] == 0xFF and inv[255] == 0xFF


def test_palette_keeps_16_of_17():
    h = np.zeros(256, np.uint64)
    for i, e in enumerate(range(100, 117)):
        h[e] = 1000 - i          # 17 exponents, strictly decreasing counts
    pal, inv = O.palette(h)
    assert list(pal) == list(range(100, 116))
    assert inv[116] == 0xFF


# --------------------------------------------------------------------------
# verbatim groups and the verbatim store
# --------------------------------------------------------------------------
def _constructed_matrix():
    """4 x 128 matrix (8 groups of 64).  16 common exponents 110..125 fill
    everything; group 1 and group 6 each get one element of exponent 200,
    which occurs twice in total and so is outside the palette."""
    N, K = 4, 128
    rng = np.random.default_rng(11)
    ex = rng.integers(110, 126, N * K)
    ex[64 + 17] = 200          # group 1 (row 0, cols 64..127)
    ex[6 * 64 + 63] = 200      # group 6 (row 3, cols 0..63)
    w = (ex.astype(np.uint16) << 7) | rng.integers(0, 128, N * K).astype(np.uint16)
    return w.reshape(N, K), ex


def test_verbatim_constructed():
    W, ex = _constructed_matrix()
    b = O.compress(W)
    assert b["V"] == 2
    assert list(b["verb"]) == [0, 1, 0, 0, 0, 0, 1, 0]
    assert b["vbits"].tolist() == [(1 << 1) | (1 << 6)]
    assert b["vpre"].tolist() == [0]
    assert np.array_equal(b["vexp"][:64], ex[64:128].astype(np.uint8))
    assert np.array_equal(b["vexp"][64:], ex[384:448].astype(np.uint8))
    # vcol: word kt*NW + n/32, NW = 4; group 1 = (n=0, kt=1); group 6 = (n=3, kt=0)
    vcol = b["vcol"].reshape(2, 4)
    assert vcol[0].tolist() == [1 << 3, 0, 0, 0]
    assert vcol[1].tolist() == [1 << 0, 0, 0, 0]
    # symbols are 0 across both verbatim groups, palette indices elsewhere
    s = b["symbols"]
    assert not s[64:128].any() and not s[384:448].any()
    assert np.array_equal(b["palette"][s[:64]], ex[:64].astype(np.uint8))


def test_verbatim_matches_rule_on_small_matrix():
    W, _ = S.small_matrix()
    b = O.compress(W)
    e, _ = O.split(W)
    pal = set(b["palette"].tolist())
    expect = np.array([any(int(x) not in pal for x in e[g * 64:(g + 1) * 64]) for g in range(0, b["G"], 1)])
    assert np.array_equal(b["verb"].astype(bool), expect)
    # the 82 forced groups (exponent + 12) must all be verbatim
    assert b["V"] >= 82


# --------------------------------------------------------------------------
# Huffman lengths
# --------------------------------------------------------------------------
def _kraft(lengths):
    return sum(Fraction(1, 2 ** int(l)) for l in lengths if l)


def _cost(freq, lengths):
    return int(sum(int(f) * int(l) for f, l in zip(freq, lengths)))


def test_clrs_example():
    rows = _read_golden("clrs_huffman.txt")
    cost = int([r for r in rows if r[0] == "cost"][0][1])
    syms = [r for r in rows if r[0] != "cost"]
    freq = np.zeros(16, np.uint64)
    expect = np.zeros(16, np.uint8)
    for s, f, l in syms:
        freq[int(s)] = int(f)
        expect[int(s)] = int(l)
    ln = O.code_lengths(freq, 12)
    assert _cost(freq, ln) == cost
    assert np.array_equal(ln, expect)
    assert _kraft(ln) == 1


def _textbook_huffman_cost(freq):
    """Plain (unlimited) Huffman cost with a heap -- an independent routine."""
    h = [int(f) for f in freq if f > 0]
    if len(h) == 1:
        return h[0]
    heapq.heapify(h)
    cost = 0
    while len(h) > 1:
        a = heapq.heappop(h)
        b = heapq.heappop(h)
        cost += a + b
        heapq.heappush(h, a + b)
    return cost


def _brute_min_cost(freq, lmax):
    used = [f for f in freq if f > 0]
    best = None
    for lens in itertools.product(range(1, lmax + 1), repeat=len(used)):
        if sum(Fraction(1, 2 ** l) for l in lens) <= 1:
            c = sum(f * l for f, l in zip(used, lens))
            best = c if best is None else min(best, c)
    return best


@pytest.mark.parametrize("seed", range(12))
def test_package_merge_optimal_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 7))
    lmax = int(rng.integers(max(1, math.ceil(math.log2(n))), 6))
    freq = np.zeros(16, np.uint64)
    pos = rng.choice(16, n, replace=False)
    freq[pos] = rng.integers(1, 60, n) ** int(rng.integers(1, 3))
    ln = O.code_lengths(freq, lmax)
    assert int(ln.max()) <= lmax
    assert _kraft(ln) == 1
    assert all((ln[i] > 0) == (freq[i] > 0) for i in range(16))
    assert _cost(freq, ln) == _brute_min_cost([int(f) for f in freq], lmax)


def test_length_limit_binds_on_fibonacci():
    fib = [1, 1]
    while len(fib) < 16:
        fib.append(fib[-1] + fib[-2])
    freq = np.array(fib, np.uint64)
    free = O.code_lengths(freq, 31)
    assert _cost(freq, free) == _textbook_huffman_cost(fib)
    assert int(free.max()) == 15
    lim = O.code_lengths(freq, 12)
    assert int(lim.max()) == 12
    assert _kraft(lim) == 1
    assert _cost(freq, lim) > _cost(freq, free)


def _package_merge_py(freq, lmax, leaf_first):
    """Independent package-merge in Python with a switchable tie rule: on
    equal weight a leaf goes before a package (leaf_first) or after it."""
    used = sorted([s for s in range(len(freq)) if freq[s] > 0], key=lambda s: (freq[s], s))
    leaves = [(int(freq[s]), {s: 1}) for s in used]
    lst = list(leaves)
    for _ in range(2, lmax + 1):
        pk = []
        for i in range(len(lst) // 2):
            (wa, ca), (wb, cb) = lst[2 * i], lst[2 * i + 1]
            c = dict(ca)
            for k, v in cb.items():
                c[k] = c.get(k, 0) + v
            pk.append((wa + wb, c))
        out, i, j = [], 0, 0
        while i < len(leaves) or j < len(pk):
            if i >= len(leaves):
                take_leaf = False
            elif j >= len(pk):
                take_leaf = True
            else:
                take_leaf = leaves[i][0] <= pk[j][0] if leaf_first else leaves[i][0] < pk[j][0]
            if take_leaf:
                out.append(leaves[i])
                i += 1
            else:
                out.append(pk[j])
                j += 1
        lst = out
    lengths = [0] * len(freq)
    for _, c in lst[:2 * (len(used) - 1)]:
        for k, v in c.items():
            lengths[k] += v
    return lengths


def test_package_merge_tie_rule_hand_derived():
    """tests/golden/package_merge_tie.txt: a leaf and a package of equal
    weight meet; leaf-first gives 2,2,2,2 and package-first 3,3,2,1 at the
    same cost, so this pins the tie rule (cost-only checks cannot)."""
    rows = _read_golden("package_merge_tie.txt")
    lmax = int([r for r in rows if r[0] == "lmax"][0][1])
    cost = int([r for r in rows if r[0] == "cost"][0][1])
    syms = [r for r in rows if r[0] not in ("lmax", "cost")]
    freq = np.zeros(16, np.uint64)
    leaf_first = np.zeros(16, np.uint8)
    pkg_first = np.zeros(16, np.uint8)
    for s, f, a, b in syms:
        freq[int(s)], leaf_first[int(s)], pkg_first[int(s)] = int(f), int(a), int(b)
    ln = O.code_lengths(freq, lmax)
    assert ln.tolist() == leaf_first.tolist()
    assert ln.tolist() != pkg_first.tolist()
    assert _cost(freq, leaf_first) == _cost(freq, pkg_first) == cost
    assert _kraft(pkg_first) == 1 and _kraft(leaf_first) == 1
    # the independent implementation reproduces both hand-derived columns
    assert _package_merge_py(freq.tolist(), lmax, True) == leaf_first.tolist()
    assert _package_merge_py(freq.tolist(), lmax, False) == pkg_first.tolist()


def test_package_merge_tie_rule_fibonacci():
    """Fibonacci frequencies at the 12-bit limit: the two tie rules give
    different optimal length vectors; the oracle gives the leaf-first one."""
    fib = [1, 1]
    while len(fib) < 16:
        fib.append(fib[-1] + fib[-2])
    leaf_first = [12, 12, 11, 10, 9, 8, 7, 6, 5, 4, 4, 4, 3, 3, 2, 2]
    pkg_first = [12, 12, 12, 12, 11, 11, 10, 10, 8, 7, 6, 5, 4, 3, 2, 1]
    assert _package_merge_py(fib, 12, True) == leaf_first
    assert _package_merge_py(fib, 12, False) == pkg_first
    assert _cost(fib, leaf_first) == _cost(fib, pkg_first)
    assert O.code_lengths(np.array(fib, np.uint64), 12).tolist() == leaf_first


def test_degenerate_alphabets():
    f = np.zeros(16, np.uint64)
    f[9] = 1000
    ln = O.code_lengths(f, 12)
    assert ln.tolist() == [0] * 9 + [1] + [0] * 6
    f[2] = 1
    ln = O.code_lengths(f, 12)
    assert ln[2] == 1 and ln[9] == 1 and int(ln.sum()) == 2


def test_rfc1951_canonical_codes():
    rows = _read_golden("rfc1951_canonical.txt")
    lens = np.zeros(16, np.uint8)
    for s, l, _ in rows:
        lens[int(s)] = int(l)
    codes = O.canonical_codes(lens)
    for s, l, c in rows:
        assert format(int(codes[int(s)]), "0%db" % int(l)) == c


# --------------------------------------------------------------------------
# encode / decode
# --------------------------------------------------------------------------
def test_tiny_hand_derived_stream():
    rows = {r[0]: r[1:] for r in _read_golden("tiny_1x64.txt")}
    ex = [120] * 32 + [121] * 16 + [122] * 8 + [123] * 8
    W = (np.array(ex, np.uint16) << 7).reshape(1, 64)
    b = O.compress(W)
    assert b["palette"].tolist() == [int(x) for x in rows["palette"]]
    assert b["code_len"].tolist() == [int(x) for x in rows["code_len"]]
    assert b["total_bits"] == int(rows["total_bits"][0])
    assert [format(int(x), "08X") for x in b["stream"]] == rows["stream"]
    expect_idx = []
    for tok in rows["idx"]:
        byte, rep = tok.split("x")
        expect_idx += [int(byte, 16)] * int(rep)
    assert b["idx"].tolist() == expect_idx
    assert b["chunk_off"].tolist() == [0] and b["seg_rel"].tolist() == [0]
    assert b["V"] == 0
    assert np.array_equal(O.decode_full(b), W)


def test_nibble_order_hand_derived():
    """tests/golden/nibble_order_1x64.txt: symbols 0,1,2,3 repeating give
    index bytes 0x10, 0x32 (element 2j in the low nibble); the swapped order
    would give 0x01, 0x23."""
    rows = {r[0]: r[1:] for r in _read_golden("nibble_order_1x64.txt")}
    ex = [120 + (k % 4) for k in range(64)]
    W = (np.array(ex, np.uint16) << 7).reshape(1, 64)
    b = O.compress(W)
    assert b["palette"].tolist() == [int(x) for x in rows["palette"]]
    assert b["code_len"].tolist() == [int(x) for x in rows["code_len"]]
    assert b["total_bits"] == int(rows["total_bits"][0])
    assert [format(int(x), "08X") for x in b["stream"]] == rows["stream"]
    expect_idx = []
    for tok in rows["idx"]:
        byte, rep = tok.split("x")
        expect_idx += [int(byte, 16)] * int(rep)
    assert b["idx"].tolist() == expect_idx
    assert b["idx"][:2].tolist() == [0x10, 0x32]
    assert np.array_equal(O.transcode(b), b["idx"])
    assert np.array_equal(O.decode_full(b), W)


def _py_decode(stream, lengths, start, count):
    """Independent bit-walking decoder: builds the code table from the
    canonical rule and matches prefixes with a dict."""
    codes = O.canonical_codes(lengths)
    table = {(int(l), int(c)): s for s, (l, c) in enumerate(zip(lengths, codes)) if l}
    out, p = [], start
    for _ in range(count):
        v, l = 0, 0
        while True:
            bit = (int(stream[p // 32]) >> (31 - p % 32)) & 1
            v, l, p = (v << 1) | bit, l + 1, p + 1
            if (l, v) in table:
                out.append(table[(l, v)])
                break
            assert l <= 12
    return out, p


def test_segment_offsets_independent_decoder():
    W, _ = S.small_matrix()
    b = O.compress(W)
    s = b["symbols"]
    nseg = b["seg_rel"].size
    assert nseg == (s.size + 255) // 256
    for j in list(range(0, 20)) + list(range(nseg - 5, nseg)):
        start = int(b["chunk_off"][j // 16]) + int(b["seg_rel"][j])
        cnt = min(256, s.size - 256 * j)
        got, _ = _py_decode(b["stream"], b["code_len"], start, cnt)
        assert got == s[256 * j:256 * j + cnt].tolist()
    # offsets are the running sum of code lengths
    bitpos = np.concatenate([[0], np.cumsum(b["code_len"][s].astype(np.int64))])
    starts = b["chunk_off"][np.arange(nseg) // 16].astype(np.int64) + b["seg_rel"].astype(np.int64)
    assert np.array_equal(starts, bitpos[np.arange(nseg) * 256])
    assert b["total_bits"] == bitpos[-1]
    assert b["stream"].size == (b["total_bits"] + 31) // 32 + 2


def test_round_trip_small_matrix():
    W, _ = S.small_matrix()
    b = O.compress(W)
    assert np.array_equal(O.decode_full(b), W)
    e, _ = O.split(W)
    assert np.array_equal(O.decode_exponent(b), e)
    assert np.array_equal(O.transcode(b), b["idx"])


def test_round_trip_every_bf16_pattern():
    W = S.all_bf16_patterns()
    b = O.compress(W)
    assert np.array_equal(O.decode_full(b), W)
    # row r holds patterns 64r..64r+63, which share one exponent, (r>>1)&0xFF;
    # every exponent occurs 256 times, so the palette is 0..15 by the tie rule
    # and exactly the 64 rows with exponents 0..15 escape the verbatim store
    assert b["palette"].tolist() == list(range(16))
    assert b["V"] == 960


def test_single_exponent_matrix():
    W = (np.full((3, 128), 127, np.uint16) << 7) | np.arange(3 * 128, dtype=np.uint16).reshape(3, 128) % 128
    b = O.compress(W)
    assert b["code_len"][0] == 1 and int(b["code_len"].sum()) == 1
    assert b["total_bits"] == 3 * 128
    assert np.array_equal(O.decode_full(b), W)


# --------------------------------------------------------------------------
# Gaussian closed form and the page's figures
# --------------------------------------------------------------------------
def _bin_mass(e, sigma):
    """P(exponent == e) for |w|, w ~ N(0, sigma) rounded to BF16 (RNE): the
    rounded value has exponent e iff 2^(e-127)(1-2^-9) <= |w| < 2^(e-126)(1-2^-9)."""
    lo = 2.0 ** (e - 127) * (1 - 2.0 ** -9)
    hi = 2.0 ** (e - 126) * (1 - 2.0 ** -9)
    return math.erf(hi / (sigma * math.sqrt(2))) - math.erf(lo / (sigma * math.sqrt(2)))


def test_gaussian_exponent_statistics():
    sigma = 0.02
    W = S.gaussian_weight(1024, 4096, seed=123, std=sigma)
    n = W.size
    b = O.compress(W)
    h = b["hist"].astype(np.float64)
    for e in range(100, 130):
        p = _bin_mass(e, sigma)
        sd = math.sqrt(n * p * (1 - p)) + 1.0
        assert abs(h[e] - n * p) <= 5 * sd, (e, h[e], n * p)
    assert sorted(b["palette"].tolist()) == list(range(108, 124))
    cover = h[b["palette"]].sum() / n
    assert cover > 0.99                        # page: top 16 cover > 99%
    assert abs(cover - (1 - 7.6e-5)) < 3e-5    # closed form at sigma = 0.02
    p = h[h > 0] / n
    H = float(-(p * np.log2(p)).sum())
    assert abs(H - 2.545) < 0.01               # closed form; page: ~2.6 bits
    f = b["freq"].astype(np.float64)
    q = f[f > 0] / f.sum()
    Hs = float(-(q * np.log2(q)).sum())
    mean = b["total_bits"] / n
    assert Hs <= mean < Hs + 1
    assert abs(mean - 2.59) < 0.03


def test_compression_ratio_near_page_figure():
    W = S.gaussian_weight(256, 4096, seed=7)
    b = O.compress(W)
    huff_bytes = (b["sm"].nbytes + b["stream"].nbytes + b["chunk_off"].nbytes + b["seg_rel"].nbytes
                  + b["vbits"].nbytes + b["vpre"].nbytes + b["vexp"].nbytes)
    ratio = huff_bytes / (2 * W.size)
    # page: ~30% saving on MLP weights -> roughly two thirds of the BF16 bytes
    assert 0.64 < ratio < 0.70


# --------------------------------------------------------------------------
# GEMM reference
# --------------------------------------------------------------------------
def _frac(bits):
    return Fraction(float(S.bits_to_float(np.array([bits], np.uint16))[0]))


def test_gemm_exact_tiny():
    X = S.activations(2, 64, seed=3)
    W = S.gaussian_weight(3, 64, seed=4)
    R = O.gemm(X, W, "f64")
    for m in range(2):
        for n in range(3):
            exact = sum(_frac(X[m, k]) * _frac(W[n, k]) for k in range(64))
            assert abs(Fraction(R[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_gemm_matches_library_matmul_and_f32_bound():
    X = S.activations(5, 256, seed=8)
    W = S.gaussian_weight(7, 256, seed=9)
    R = O.gemm(X, W, "f64")
    ref = S.bits_to_float(X).astype(np.float64) @ S.bits_to_float(W).astype(np.float64).T
    assert np.allclose(R, ref, rtol=1e-12, atol=1e-14)
    R32 = O.gemm(X, W, "f32")
    absdot = np.abs(S.bits_to_float(X).astype(np.float64)) @ np.abs(S.bits_to_float(W).astype(np.float64)).T
    assert np.all(np.abs(R32 - R) <= 256 * 2.0 ** -24 * absdot + 1e-30)
    assert O.gemm_one(X, W, 3, 5) == R[3, 5]


# --------------------------------------------------------------------------
# SwiGLU (the MLP's activation between gate/up and down)
# --------------------------------------------------------------------------
def test_swiglu_identities():
    z = np.array([0.0, 0.25, -0.25, 1.0, -1.0, 3.5, -3.5, 12.0, -12.0, 40.0, -40.0])
    ones = np.ones_like(z)
    h = O.swiglu(z, ones)
    # silu(0) = 0; silu(z) - silu(-z) = z (z s(z) + z s(-z) = z)
    assert h[0] == 0.0
    hn = O.swiglu(-z, ones)
    assert np.allclose(h - hn, z, rtol=1e-14, atol=1e-14)
    # an independent form: silu(z) = z/2 * (1 + tanh(z/2))
    for zi, hi in zip(z, h):
        assert abs(hi - zi / 2 * (1 + math.tanh(zi / 2))) <= 1e-14 * max(1.0, abs(zi))
    # far tails: silu(40) = 40 to double precision, silu(-40) = -40 e^-40 (1 + O(e^-40))
    assert h[-2] == 40.0
    assert abs(h[-1] / (-40.0 * math.exp(-40.0)) - 1) < 1e-12
    # the up product scales the result linearly (the gate does not)
    u = np.array([2.0, -3.0, 0.5, 8.0, -0.125, 1.0, 1.0, 4.0, 4.0, 1.0, 1.0])
    assert np.array_equal(O.swiglu(z, u), h * u)
    assert O.swiglu(np.array([1.0]), np.array([2.0]))[0] == pytest.approx(2.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
