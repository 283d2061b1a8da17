"""Pins for the CPU oracle: facts that do not come from the oracle's own code.

Each test states what fixes the expected value: a hand-worked fixture (with its
source under tests/golden/), a closed form, an invariant of optimal prefix codes,
brute force on tiny alphabets, a textbook Huffman built here with heapq, or a
library routine (torch's fp32->bf16 conversion, NumPy's float64 matrix product).
"""
import heapq
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads


def _golden_rows(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


# ---------------------------------------------------------------- canonical codes

def test_canonical_codes_rfc1951_example(golden_dir):
    rows = [r.split() for r in _golden_rows(golden_dir, "canonical_rfc1951.txt")]
    lengths = np.zeros(256, np.uint8)
    for sym, ln, _ in rows:
        lengths[int(sym)] = int(ln)
    codes = oracle.canonical_codes(lengths)
    for sym, ln, bits in rows:
        assert format(int(codes[int(sym)]), f"0{int(ln)}b") == bits


def test_canonical_codes_prefix_free_and_ordered():
    rng = np.random.default_rng(7)
    for _ in range(50):
        hist = rng.integers(0, 50, size=256)
        hist[rng.integers(0, 256)] += 1
        lengths = oracle.code_lengths(hist, 16)
        codes = oracle.canonical_codes(lengths)
        words = sorted((format(int(codes[s]), f"0{int(lengths[s])}b"), int(lengths[s]), s)
                       for s in range(256) if lengths[s])
        # prefix-free: in lexicographic order a prefix would sit right before its extension
        for (a, _, _), (b, _, _) in zip(words, words[1:]):
            assert not b.startswith(a)
        # canonical: lexicographic order == (length, symbol) order
        assert [s for _, _, s in words] == [s for _, _, s in sorted(words, key=lambda t: (t[1], t[2]))]


# ---------------------------------------------------------------- code lengths

def _cost(hist, lengths):
    return int(sum(int(h) * int(l) for h, l in zip(hist, lengths)))


def _kraft_scaled(lengths, lmax):
    return sum(1 << (lmax - int(l)) for l in lengths if l)


def test_code_lengths_handworked(golden_dir):
    for row in _golden_rows(golden_dir, "lengths_handworked.txt"):
        lmax, counts, expect, cost = [p.split() for p in row.split("|")]
        hist = np.array([int(c) for c in counts], np.int64)
        got = oracle.code_lengths(hist, int(lmax[0]))
        assert [int(v) for v in got] == [int(v) for v in expect], row
        assert _cost(hist, got) == int(cost[0]), row


def _brute_force_cost(counts, lmax):
    """Minimum cost over all length vectors with Kraft <= 1 and lengths <= lmax."""
    active = sorted((c for c in counts if c > 0), reverse=True)
    m = len(active)
    if m == 1:
        return active[0]
    best = None
    for lens in itertools.combinations_with_replacement(range(1, lmax + 1), m):
        if sum(2.0 ** -l for l in lens) <= 1.0 + 1e-12:
            c = sum(a * l for a, l in zip(active, lens))
            best = c if best is None else min(best, c)
    return best


@pytest.mark.parametrize("seed", range(40))
def test_code_lengths_match_brute_force(seed):
    rng = np.random.default_rng(1000 + seed)
    m = int(rng.integers(2, 9))
    hist = np.zeros(16, np.int64)
    syms = rng.choice(16, size=m, replace=False)
    hist[syms] = rng.integers(1, 60, size=m) ** int(rng.integers(1, 3))
    lo = max(1, math.ceil(math.log2(m)))
    for lmax in range(lo, 8):
        got = oracle.code_lengths(hist, lmax)
        assert int(got.max()) <= lmax
        assert _kraft_scaled(got, lmax) == (1 << lmax)          # complete code
        assert _cost(hist, got) == _brute_force_cost(hist, lmax), (hist, lmax, got)


def _textbook_huffman_lengths(hist):
    """Unlimited Huffman code lengths with a heap (Huffman 1952)."""
    items = [(int(h), i, (i,)) for i, h in enumerate(hist) if h > 0]
    lengths = np.zeros(len(hist), np.int64)
    if len(items) == 1:
        lengths[items[0][2][0]] = 1
        return lengths
    heapq.heapify(items)
    tick = len(hist)
    while len(items) > 1:
        w1, _, s1 = heapq.heappop(items)
        w2, _, s2 = heapq.heappop(items)
        for s in s1 + s2:
            lengths[s] += 1
        heapq.heappush(items, (w1 + w2, tick, s1 + s2))
        tick += 1
    return lengths


def _entropy_np(hist):
    p = hist[hist > 0] / hist.sum()
    return float(-(p * np.log2(p)).sum())


@pytest.mark.parametrize("seed", range(30))
def test_code_lengths_vs_textbook_huffman(seed):
    rng = np.random.default_rng(2000 + seed)
    kind = seed % 3
    if kind == 0:
        hist = rng.integers(0, 1000, size=256)
    elif kind == 1:
        hist = np.floor(1e6 * np.exp(-0.5 * ((np.arange(256) - 128) / rng.uniform(2, 30)) ** 2))
    else:
        hist = np.floor(1e6 * np.exp(-np.abs(np.arange(16) - 8) / rng.uniform(0.3, 3)))
    hist = hist.astype(np.int64)
    if hist.sum() == 0:
        hist[0] = 1
    huff = _textbook_huffman_lengths(hist)
    for lmax in (12, 16, 24):
        if (hist > 0).sum() > (1 << lmax):
            continue
        got = oracle.code_lengths(hist, lmax)
        assert int(got.max()) <= lmax
        if (hist > 0).sum() >= 2:
            assert _kraft_scaled(got, lmax) == (1 << lmax)
        H = _entropy_np(hist)
        avg = _cost(hist, got) / hist.sum()
        assert avg >= H - 1e-12
        if huff.max() <= lmax:
            assert _cost(hist, got) == _cost(hist, huff)        # unlimited optimum reached
            assert avg < H + 1.0
        else:
            assert _cost(hist, got) >= _cost(hist, huff)


def test_code_lengths_limit_errors():
    with pytest.raises(oracle.OracleError):
        oracle.code_lengths(np.ones(256, np.int64), 7)          # 256 symbols need >= 8 bits
    got = oracle.code_lengths(np.ones(256, np.int64), 8)
    assert (got == 8).all()                                      # uniform over 2^k -> all k


# ---------------------------------------------------------------- quantization

def test_quantize_handworked(golden_dir):
    for row in _golden_rows(golden_dir, "quant_handworked.txt"):
        head, ws, scale, zero, codes = [p.split() for p in row.split("|")]
        bits, mode = int(head[0]), int(head[1])
        w = np.array([float(v) for v in ws], np.float32)
        q, s, z, _ = oracle.quantize(w, bits, mode)
        assert s == float(scale[0]), row
        assert z == int(zero[0]), row
        assert [int(v) for v in q] == [int(v) for v in codes], row


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("kind", ["t4", "laplace", "uniform", "skew"])
def test_asymmetric_quantization_properties(bits, kind):
    w = workloads.small_tensor(kind, 64, 96, seed=bits).reshape(-1)
    q, s, z, scheme = oracle.quantize(w, bits, oracle.MODE_ASYM)
    qmax = (1 << bits) - 1
    assert scheme == oracle.SCHEME_ASYM
    assert q[np.argmin(w)] == 0                                  # round(x) + round(-x) = 0
    assert q[np.argmax(w)] >= qmax - 1
    order = np.argsort(w, kind="stable")
    assert (np.diff(q[order].astype(int)) >= 0).all()            # monotone
    rec = (q.astype(np.float64) - z) * s
    inside = (w >= (0 - z) * s) & (w <= (qmax - z) * s)
    assert np.all(np.abs(rec - w)[inside] <= 0.5 * s * (1 + 1e-6) + 1e-7 * np.abs(w[inside]))
    assert abs(s - (float(w.max()) - float(w.min())) / qmax) <= 1e-7 * s


@pytest.mark.parametrize("bits", [4, 8])
def test_unsigned_quantization_properties(bits):
    w = workloads.small_tensor("shifted", 50, 70, seed=3).reshape(-1)
    q, s, z, scheme = oracle.quantize(w, bits, oracle.MODE_UNSIGNED)
    qmax = (1 << bits) - 1
    assert scheme == oracle.SCHEME_UNSIGNED and z == 0
    assert q[np.argmax(w)] == qmax and q[np.argmin(w)] == 0      # min is exactly 0 here
    assert np.all(np.abs(q * np.float64(s) - w) <= 0.5 * s * (1 + 1e-6))
    with pytest.raises(oracle.OracleError):
        oracle.quantize(np.array([-1.0, 1.0], np.float32), bits, oracle.MODE_UNSIGNED)


def test_auto_picks_lower_entropy():
    # negative values: unsigned is not eligible, AUTO == asymmetric
    w = workloads.small_tensor("t4", 40, 40, seed=1)
    assert oracle.quantize(w, 8, oracle.MODE_AUTO)[3] == oracle.SCHEME_ASYM
    # min > 0 and two close values: unsigned's coarser grid merges them (2 codes vs 3)
    w = np.array([0.51, 0.511, 1.0, 0.51, 0.511, 1.0], np.float32)
    qa = oracle.quantize(w, 8, oracle.MODE_ASYM)[0]
    qu = oracle.quantize(w, 8, oracle.MODE_UNSIGNED)[0]
    ha, hu = _entropy_np(np.bincount(qa, minlength=256)), _entropy_np(np.bincount(qu, minlength=256))
    assert hu < ha
    q, s, z, scheme = oracle.quantize(w, 8, oracle.MODE_AUTO)
    assert scheme == oracle.SCHEME_UNSIGNED and (q == qu).all()
    # shifted tensors (min == 0): both schemes coincide, the tie goes to unsigned
    w = workloads.small_tensor("shifted", 30, 30, seed=2)
    assert oracle.quantize(w, 8, oracle.MODE_AUTO)[3] == oracle.SCHEME_UNSIGNED
    # in every case AUTO's entropy is the lower of the two candidates
    for kind in ("positive", "shifted", "t4"):
        w = workloads.small_tensor(kind, 33, 65, seed=9)
        qauto = oracle.quantize(w, 8, oracle.MODE_AUTO)[0]
        cands = [oracle.quantize(w, 8, oracle.MODE_ASYM)[0]]
        if w.min() >= 0:
            cands.append(oracle.quantize(w, 8, oracle.MODE_UNSIGNED)[0])
        ents = [_entropy_np(np.bincount(c, minlength=256)) for c in cands]
        assert _entropy_np(np.bincount(qauto, minlength=256)) <= min(ents) + 1e-12


def test_quantize_special_cases():
    q, s, z, _ = oracle.quantize(np.full(10, -0.375, np.float32), 8, oracle.MODE_AUTO)
    assert (q == 1).all() and s == -0.375 and z == 0
    q, s, z, _ = oracle.quantize(np.zeros(10, np.float32), 4, oracle.MODE_AUTO)
    assert (q == 0).all() and s == 1.0 and z == 0
    q, s, z, _ = oracle.quantize(np.zeros(0, np.float32), 8, oracle.MODE_ASYM)
    assert q.size == 0
    for bad in (np.nan, np.inf, -np.inf):
        with pytest.raises(oracle.OracleError):
            oracle.quantize(np.array([0.0, bad], np.float32), 8, oracle.MODE_ASYM)


# ---------------------------------------------------------------- dequant (bf16 RNE)

def _torch_bf16_bits(f32):
    return torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_dequant_matches_torch_bf16_rounding():
    rng = np.random.default_rng(11)
    for bits in (4, 8):
        q = rng.integers(0, 1 << bits, size=20000).astype(np.uint8)
        for s, z in ((0.0303817, 8), (1e-3, 128), (-0.375, 0), (3.7e-5, -200), (1.0, 0)):
            s = float(np.float32(s))
            got = oracle.dequant_bf16(q, s, z)
            prod = (q.astype(np.int64) - z).astype(np.float32) * np.float32(s)   # IEEE fp32 multiply
            assert (got == _torch_bf16_bits(prod)).all()


def test_dequant_ties_to_even():
    # (q - z) * 1.0 with q - z chosen so that the fp32 value sits exactly halfway between
    # two bf16 values: 257 = 0x43808000 (tie, even below), 259 = 0x43818000 (tie, odd below)
    got = oracle.dequant_bf16(np.array([1, 3], np.uint8), 1.0, -256)
    assert list(got) == [0x4380, 0x4382]
    assert list(got) == list(_torch_bf16_bits(np.array([257.0, 259.0], np.float32)))


# ---------------------------------------------------------------- GEMV

def test_gemv_matches_numpy_float64():
    rng = np.random.default_rng(5)
    w = torch.from_numpy(rng.standard_normal((37, 300)).astype(np.float32)).to(torch.bfloat16)
    x = torch.from_numpy(rng.standard_normal((3, 300)).astype(np.float32)).to(torch.bfloat16)
    wb, xb = workloads.bf16_bits(w), workloads.bf16_bits(x)
    y, mag = oracle.gemv(wb, xb)
    ref = x.double().numpy() @ w.double().numpy().T
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(mag, np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T, rtol=1e-14)


# ---------------------------------------------------------------- bit layout (closed forms)

def _two_code_tensor(bits01):
    """0 -> -1.0 and 1 -> 0.875: 4-bit asymmetric gives scale 0.125, zero 8, codes 0 and 15,
    each with a 1-bit canonical code (0 -> '0', 15 -> '1')."""
    return np.where(np.asarray(bits01) == 1, 0.875, -1.0).astype(np.float32)


@pytest.mark.parametrize("lanes", [32, 64])
def test_lane_layout_closed_form(lanes):
    step = 8 * lanes
    n = 2 * step + 40                                    # two full lane steps + a ragged tail
    p = np.arange(n)
    b = ((p * 7) % 5 == 1).astype(np.uint8)
    blob = oracle.encode(_two_code_tensor(b).reshape(1, n), 4, oracle.MODE_ASYM, 12,
                         oracle.FMT_LANES, 2048, lanes=lanes)
    prm = oracle.params(blob)
    assert prm["lengths"][0] == 1 and prm["lengths"][15] == 1 and prm["lengths"].sum() == 2
    assert prm["lanes"] == lanes and prm["n_chunks"] == 1 and prm["payload_words"] == lanes
    idx = np.frombuffer(blob, np.uint64, 4, 384)
    assert list(idx) == [0, 0, lanes, n]
    words = np.frombuffer(blob, np.uint32, lanes, 384 + 32)
    for lane in range(lanes):
        seq = [int(b[q]) for t in range(3) for q in range(step * t + 8 * lane, step * t + 8 * lane + 8)
               if q < n]
        expect = 0
        for i, bit in enumerate(seq):
            expect |= bit << (31 - i)
        assert int(words[lane]) == expect, lane


@pytest.mark.parametrize("lanes", [32, 64])
def test_row_tile_layout_closed_form(lanes):
    """Row tiles of `lanes` rows by 40 columns (the last column tile 24 wide, the last row
    group ragged): with one-bit codes, word i of lane l of a tile holds bits 32i .. 32i+31
    of row l of the tile, MSB first, and lanes past the tile's last row stay zero."""
    rows, cols, kc = 2 * lanes + 6, 104, 40
    b = (((np.arange(rows)[:, None] * 5 + np.arange(cols)[None, :] * 3) % 7) < 3).astype(np.uint8)
    blob = oracle.encode(_two_code_tensor(b), 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS, lanes * kc,
                         lanes=lanes)
    prm = oracle.params(blob)
    assert prm["format"] == oracle.FMT_ROWS and prm["lanes"] == lanes
    assert prm["lengths"][0] == 1 and prm["lengths"][15] == 1 and prm["lengths"].sum() == 2
    tiles = [(g, j) for g in range(3) for j in range(3)]
    assert prm["n_chunks"] == len(tiles)
    idx = np.frombuffer(blob, np.uint64, 2 * (len(tiles) + 1), 384).reshape(-1, 2)
    words = np.frombuffer(blob, np.uint32, prm["payload_words"], 384 + 16 * (len(tiles) + 1))
    start = first = 0
    for c, (g, j) in enumerate(tiles):
        r0, c0 = g * lanes, j * kc
        nr, wd = min(lanes, rows - r0), min(kc, cols - c0)
        wc = -(-wd // 32)                                # one bit per code
        assert (int(idx[c, 0]), int(idx[c, 1])) == (start, first), c
        for lane in range(lanes):
            for i in range(wc):
                expect = 0
                if lane < nr:
                    for k in range(32):
                        if 32 * i + k < wd:
                            expect |= int(b[r0 + lane, c0 + 32 * i + k]) << (31 - k)
                assert int(words[start + lanes * i + lane]) == expect, (c, lane, i)
        start += wc * lanes
        first += nr * wd
    assert (int(idx[-1, 0]), int(idx[-1, 1])) == (start, rows * cols) and prm["payload_words"] == start


def test_single_stream_layout_closed_form():
    n = 100
    b = ((np.arange(n) * 3) % 7 < 3).astype(np.uint8)
    blob = oracle.encode(_two_code_tensor(b).reshape(10, 10), 4, oracle.MODE_ASYM, 12,
                         oracle.FMT_SINGLE, 30)
    prm = oracle.params(blob)
    assert prm["n_chunks"] == 4 and prm["payload_words"] == 4
    idx = np.frombuffer(blob, np.uint64, 10, 384).reshape(5, 2)
    assert idx[:, 0].tolist() == [0, 30, 60, 90, 100]       # bit offsets: one bit per symbol
    assert idx[:, 1].tolist() == [0, 30, 60, 90, 100]
    words = np.frombuffer(blob, np.uint32, 4, 384 + 80)
    for k in range(4):
        expect = 0
        for i in range(32):
            if 32 * k + i < n:
                expect |= int(b[32 * k + i]) << (31 - i)
        assert int(words[k]) == expect


# ---------------------------------------------------------------- encode -> decode identity

CASES = [
    ("t4", 8, oracle.MODE_ASYM, 16, oracle.FMT_SINGLE, 4096, 64, 64),
    ("t4", 8, oracle.MODE_ASYM, 16, oracle.FMT_SINGLE, 1000, 33, 65),
    ("laplace", 4, oracle.MODE_ASYM, 12, oracle.FMT_LANES, 8192, 128, 96),
    ("laplace", 4, oracle.MODE_ASYM, 12, oracle.FMT_LANES, 512, 7, 131),
    ("t4", 8, oracle.MODE_AUTO, 16, oracle.FMT_LANES, 768, 50, 51),
    ("shifted", 8, oracle.MODE_AUTO, 16, oracle.FMT_LANES, 256, 3, 300),
    ("skew", 8, oracle.MODE_ASYM, 16, oracle.FMT_LANES, 16384, 200, 100),
    ("skew", 8, oracle.MODE_ASYM, 9, oracle.FMT_LANES, 1024, 20, 100),
    ("uniform", 8, oracle.MODE_ASYM, 16, oracle.FMT_LANES, 2048, 40, 64),
    ("constant", 8, oracle.MODE_AUTO, 16, oracle.FMT_LANES, 256, 5, 77),
    ("zeros", 4, oracle.MODE_AUTO, 12, oracle.FMT_SINGLE, 50, 3, 33),
    ("two_values", 4, oracle.MODE_ASYM, 12, oracle.FMT_LANES, 256, 1, 1),
    ("t4", 4, oracle.MODE_ASYM, 4, oracle.FMT_LANES, 512, 9, 100),
    ("laplace", 4, oracle.MODE_ASYM, 12, oracle.FMT_LANES, -1024, 7, 333),    # 64 lanes
    ("t4", 8, oracle.MODE_AUTO, 16, oracle.FMT_LANES, -8192, 40, 300),        # 64 lanes
    ("laplace", 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS, 8192, 100, 1000),   # row tiles, ragged both ways
    ("t4", 8, oracle.MODE_AUTO, 16, oracle.FMT_ROWS, 4096, 70, 3072),
    ("skew", 8, oracle.MODE_ASYM, 16, oracle.FMT_ROWS, 512, 33, 24),
    ("laplace", 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS, -1024, 130, 520),   # 64-row tiles
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-b{c[1]}-f{c[4]}-c{c[5]}-{c[6]}x{c[7]}" for c in CASES])
def test_encode_decode_identity(case):
    kind, bits, mode, lmax, fmt, chunk, rows, cols = case
    lanes = 64 if chunk < 0 else 32                      # a negative chunk size marks the 64-lane cases
    chunk = abs(chunk)
    w = workloads.small_tensor(kind, rows, cols, seed=rows + cols)
    blob = oracle.encode(w, bits, mode, lmax, fmt, chunk, lanes=lanes)
    q, s, z, scheme = oracle.quantize(w, bits, mode)
    assert (oracle.decode(blob) == q).all()
    prm = oracle.params(blob)
    assert (prm["scale"], prm["zero"], prm["scheme"]) == (s, z, scheme)
    lengths = prm["lengths"][: 1 << bits]
    hist = np.bincount(q, minlength=1 << bits)
    assert int(lengths.max()) <= lmax and ((lengths > 0) == (hist > 0)).all()
    if (hist > 0).sum() >= 2:
        assert _kraft_scaled(lengths, lmax) == (1 << lmax)
    # chunk-range decode agrees with the whole decode
    if prm["n_chunks"] > 1:
        c0, c1 = 1, prm["n_chunks"]
        part = oracle.decode_chunks(blob, c0, c1)
        if fmt != oracle.FMT_ROWS:
            assert (part == q[c0 * prm["chunk_symbols"]:]).all()
        else:                                            # tiles, each row-major
            Q = q.reshape(rows, cols)
            tiles = [oracle.tile(prm, c) for c in range(c0, c1)]
            want = np.concatenate([Q[r0:r0 + nr, k0:k0 + wd].reshape(-1) for r0, k0, nr, wd in tiles])
            assert (part == want).all()


def test_empty_tensor_blob():
    blob = oracle.encode(np.zeros((0, 16), np.float32), 8, oracle.MODE_ASYM, 16, oracle.FMT_LANES, 256)
    prm = oracle.params(blob)
    assert prm["n"] == 0 and prm["n_chunks"] == 0 and prm["payload_words"] == 0
    assert oracle.decode(blob).size == 0


def test_workload_codes_statistics():
    """The 4-bit Laplace workload: the 12-bit limit binds, Kraft stays exactly 1."""
    W = workloads.get("laplace_4096x4096_u4")
    w = workloads.weights(W, W.tensors[0]).numpy()[:1024]
    q, s, z, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
    hist = np.bincount(q, minlength=16).astype(np.int64)
    lengths = oracle.code_lengths(hist, 12)
    assert _kraft_scaled(lengths, 12) == 1 << 12
    H = _entropy_np(hist)
    avg = _cost(hist, lengths) / hist.sum()
    assert H <= avg < H + 1
    assert avg >= _cost(hist, _textbook_huffman_lengths(hist)) / hist.sum()


def test_corrupted_blobs_are_rejected_or_detected():
    w = workloads.small_tensor("laplace", 64, 128, seed=4)
    blob = bytearray(oracle.encode(w, 4, oracle.MODE_ASYM, 12, oracle.FMT_SINGLE, 1024))
    q = oracle.quantize(w, 4, oracle.MODE_ASYM)[0]
    with pytest.raises(oracle.OracleError):
        oracle.decode(bytes(blob[:-8]))                        # truncated payload
    bad = bytearray(blob)
    bad[0] ^= 1
    with pytest.raises(oracle.OracleError):
        oracle.decode(bytes(bad))                              # bad magic
    bad = bytearray(blob)
    bad[384 + 16] = (bad[384 + 16] + 1) % 256                  # chunk 1 starts one bit late
    try:
        got = oracle.decode(bytes(bad))
        assert not (got == q).all()
    except oracle.OracleError:
        pass


# ---------------------------------------------------------------- consumption-order row tiles

def _co_expected_payload(q, rows, cols, bits, lanes, chunk, lengths, lmax):
    """The consumption-order layout restated in Python from its definition: each lane's
    words from its codes (canonical, MSB first); a count header; words 0-2 of every lane
    in three rows; the later words in the order a lock-step reference decoder takes them
    (lookups of at most 8 / 4 whole codes within 12 bits, or one longer code; a refill
    point before every even lookup, before every lookup when the length limit is above
    16; a lane whose taken bits reach 32 there gives back 32 and takes a word)."""
    codes = oracle.canonical_codes(lengths)
    Q = q.reshape(rows, cols)
    kc = chunk // lanes
    every = lmax > 16
    m = 8 if bits == 4 else 4
    out = []
    for g in range(-(-rows // lanes)):
        for j in range(-(-cols // kc)):
            r0, c0 = g * lanes, j * kc
            nr, wd = min(lanes, rows - r0), min(kc, cols - c0)
            lane_words, lane_lens = [], []
            for lane in range(lanes):
                bitstr = ""
                ln = []
                if lane < nr:
                    for v in Q[r0 + lane, c0:c0 + wd]:
                        bitstr += format(int(codes[v]), "0%db" % int(lengths[v]))
                        ln.append(int(lengths[v]))
                nwl = -(-len(bitstr) // 32)
                bitstr += "0" * (32 * nwl - len(bitstr))
                lane_words.append([int(bitstr[32 * i:32 * i + 32], 2) for i in range(nwl)])
                lane_lens.append(ln)
            # schedule
            state = [dict(done=0, lookups=0, c=0, taken=min(3, len(lane_words[l]))) for l in range(lanes)]
            order = []
            p = 0
            while any(state[l]["taken"] < len(lane_words[l]) for l in range(lanes)):
                for l in range(lanes):
                    s = state[l]
                    if s["taken"] >= len(lane_words[l]):
                        continue
                    while s["lookups"] < (p if every else 2 * p):
                        ln = lane_lens[l]
                        if ln[s["done"]] > 12:
                            used, k = ln[s["done"]], 1
                        else:
                            used = k = 0
                            while k < m and s["done"] + k < len(ln) and used + ln[s["done"] + k] <= 12:
                                used += ln[s["done"] + k]
                                k += 1
                        s["done"] += k
                        s["c"] += used
                        s["lookups"] += 1
                    if s["c"] >= 32:
                        s["c"] -= 32
                        order.append(lane_words[l][s["taken"]])
                        s["taken"] += 1
                p += 1
            nws = [len(w) for w in lane_words]
            cb = 1 if -(-kc * lmax // 32) <= 255 else 2
            hdr = b"".join(int(n).to_bytes(cb, "little") for n in nws)
            hdr += b"\0" * (-len(hdr) % 4)
            words = list(np.frombuffer(hdr, np.uint32))
            for r in range(3):
                words += [lane_words[l][r] if r < nws[l] else 0 for l in range(lanes)]
            words += order
            words += [0] * (-len(words) % 4)
            out.extend(words)
    return np.array(out, dtype=np.uint32)


@pytest.mark.parametrize("kind,bits,lmax,chunk,rows,cols,lanes", [
    ("laplace", 4, 12, 8192, 40, 1000, 32),
    ("t4", 8, 16, 4096, 36, 264, 32),
    ("laplace", 4, 12, 16384, 70, 512, 64),
])
def test_consumption_order_layout_restated(kind, bits, lmax, chunk, rows, cols, lanes):
    """The oracle's consumption-order payload equals the layout rebuilt from its
    definition by an independent Python statement, word for word."""
    w = workloads.small_tensor(kind, rows, cols, seed=7 + rows)
    blob = oracle.encode(w, bits, oracle.MODE_ASYM, lmax, oracle.FMT_ROWS_CO, chunk, lanes=lanes)
    prm = oracle.params(blob)
    q, _, _, _ = oracle.quantize(w, bits, oracle.MODE_ASYM)
    want = _co_expected_payload(q, rows, cols, bits, lanes, chunk, prm["lengths"], lmax)
    n_chunks = prm["n_chunks"]
    got = np.frombuffer(blob, np.uint32, prm["payload_words"], 384 + 16 * (n_chunks + 1))
    assert got.size == want.size and (got == want).all()
    assert (oracle.decode(blob) == q).all()


@pytest.mark.parametrize("lanes", [32, 64])
def test_consumption_order_closed_form(lanes):
    """One-bit codes: every lookup takes 8 codes (8 bits), so a lane's count reaches 32 at
    every second refill point: word 3 + k of every lane is taken at refill point 2k + 2,
    all lanes of the tile in lane order.  Tiles of 160 and 104 columns (5 and 4 words per
    lane), a second row group of 6 rows."""
    kc = 160
    rows, cols = lanes + 6, kc + 104
    b = (((np.arange(rows)[:, None] * 3 + np.arange(cols)[None, :] * 5) % 11) < 4).astype(np.uint8)
    blob = oracle.encode(_two_code_tensor(b), 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS_CO, lanes * kc,
                         lanes=lanes)
    prm = oracle.params(blob)
    assert prm["format"] == oracle.FMT_ROWS_CO and prm["n_chunks"] == 4
    assert prm["lengths"][0] == 1 and prm["lengths"][15] == 1 and prm["lengths"].sum() == 2
    idx = np.frombuffer(blob, np.uint64, 10, 384).reshape(-1, 2)
    words = np.frombuffer(blob, np.uint32, prm["payload_words"], 384 + 80)
    hw = lanes // 4                                       # one count byte per lane
    start = 0
    for c, (g, j) in enumerate([(0, 0), (0, 1), (1, 0), (1, 1)]):
        r0, c0 = g * lanes, j * kc
        nr, wd = min(lanes, rows - r0), min(kc, cols - c0)
        nw = -(-wd // 32)

        def lane_word(lane, i):
            e = 0
            for k in range(32):
                if 32 * i + k < wd:
                    e |= int(b[r0 + lane, c0 + 32 * i + k]) << (31 - k)
            return e

        assert int(idx[c, 0]) == start
        counts = np.frombuffer(words[start:start + hw].tobytes(), np.uint8)
        assert counts.tolist() == [nw] * nr + [0] * (lanes - nr)
        for r in range(3):
            for lane in range(lanes):
                assert int(words[start + hw + lanes * r + lane]) == (lane_word(lane, r) if lane < nr else 0)
        pos = start + hw + 3 * lanes
        for k in range(nw - 3):
            for lane in range(nr):
                assert int(words[pos]) == lane_word(lane, 3 + k), (c, k, lane)
                pos += 1
        size = hw + 3 * lanes + nr * (nw - 3)
        size += -size % 4
        assert all(int(x) == 0 for x in words[pos:start + size])
        start += size
    assert int(idx[-1, 0]) == start == prm["payload_words"]


def _long_code_tensor(rows, cols, seed):
    """8-bit codes with geometric frequencies (symbol k about 2^-k of the weights), so
    that the Huffman lengths reach past 16 bits under a 20-bit limit."""
    n = rows * cols
    counts = [max(1, n >> (k + 1)) for k in range(24)]
    vals = np.concatenate([np.full(c, k, np.float32) for k, c in enumerate(counts)])
    vals = np.concatenate([vals, np.full(max(0, n - vals.size), 0, np.float32)])[:n]
    vals[-1] = 255.0                                     # scale 1, zero 0: q = w
    rng = np.random.default_rng(seed)
    rng.shuffle(vals)
    return vals.reshape(rows, cols)


CO_CASES = [
    ("laplace", 4, oracle.MODE_ASYM, 12, 8192, 100, 1000, 32),
    ("t4", 8, oracle.MODE_AUTO, 16, 4096, 70, 3072, 32),
    ("skew", 8, oracle.MODE_ASYM, 16, 512, 33, 24, 32),
    ("laplace", 4, oracle.MODE_ASYM, 12, 1024, 130, 520, 64),
    ("uniform", 8, oracle.MODE_ASYM, 16, 16384, 40, 1024, 32),
    ("two_values", 4, oracle.MODE_ASYM, 12, 256, 1, 8, 32),
]


@pytest.mark.parametrize("case", CO_CASES, ids=[f"{c[0]}-b{c[1]}-c{c[4]}-{c[5]}x{c[6]}-L{c[7]}" for c in CO_CASES])
def test_consumption_order_identity(case):
    kind, bits, mode, lmax, chunk, rows, cols, lanes = case
    w = workloads.small_tensor(kind, rows, cols, seed=rows + cols)
    blob = oracle.encode(w, bits, mode, lmax, oracle.FMT_ROWS_CO, chunk, lanes=lanes)
    q, _, _, _ = oracle.quantize(w, bits, mode)
    assert (oracle.decode(blob) == q).all()
    static = oracle.encode(w, bits, mode, lmax, oracle.FMT_ROWS, chunk, lanes=lanes)
    assert oracle.params(blob)["lengths"].tolist() == oracle.params(static)["lengths"].tolist()
    prm = oracle.params(blob)
    if prm["n_chunks"] > 1:
        Q = q.reshape(rows, cols)
        part = oracle.decode_chunks(blob, 1, prm["n_chunks"])
        tiles = [oracle.tile(prm, c) for c in range(1, prm["n_chunks"])]
        want = np.concatenate([Q[r0:r0 + nr, k0:k0 + wd].reshape(-1) for r0, k0, nr, wd in tiles])
        assert (part == want).all()


def test_consumption_order_long_codes():
    """Length limit 20 (codes longer than 16 bits): refill points before every lookup."""
    w = _long_code_tensor(256, 1024, 5)
    blob = oracle.encode(w, 8, oracle.MODE_ASYM, 20, oracle.FMT_ROWS_CO, 8192, lanes=32)
    prm = oracle.params(blob)
    assert int(prm["lengths"].max()) > 16
    q, _, _, _ = oracle.quantize(w, 8, oracle.MODE_ASYM)
    assert (oracle.decode(blob) == q).all()
    want = _co_expected_payload(q, 256, 1024, 8, 32, 8192, prm["lengths"], 20)
    got = np.frombuffer(blob, np.uint32, prm["payload_words"], 384 + 16 * (prm["n_chunks"] + 1))
    assert (got == want).all()


def test_consumption_order_smaller_than_padded_lanes():
    """On a Mistral-shaped 4-bit tile set the consumption order stores fewer words than
    lanes padded to the tile's longest (the point of the layout)."""
    W = workloads.get("mistral_7b_u4")
    w = workloads.weights(W, W.tensors[1]).numpy()[:128]
    co = oracle.params(oracle.encode(w, 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS_CO, 8192))["payload_words"]
    st = oracle.params(oracle.encode(w, 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS, 8192))["payload_words"]
    assert co < 0.97 * st, (co, st)


def test_consumption_order_corrupt_counts():
    w = workloads.small_tensor("laplace", 64, 512, seed=3)
    blob = bytearray(oracle.encode(w, 4, oracle.MODE_ASYM, 12, oracle.FMT_ROWS_CO, 8192))
    prm = oracle.params(bytes(blob))
    base = 384 + 16 * (prm["n_chunks"] + 1)
    q, _, _, _ = oracle.quantize(w, 4, oracle.MODE_ASYM)
    for extra, must_raise in ((40, True), (200, True), (1, False)):
        bad = bytearray(blob)
        bad[base + 5] = (bad[base + 5] + extra) & 0xFF    # lane 5 claims more words than it has
        if must_raise:                                    # it runs out of codes, or past the limit
            with pytest.raises(oracle.OracleError):
                oracle.decode(bytes(bad))
        else:                                             # every later word shifts: never the same codes
            try:
                assert not (oracle.decode(bytes(bad)) == q).all()
            except oracle.OracleError:
                pass
