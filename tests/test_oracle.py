"""Pins for the CPU oracle, each against something other than the oracle.

- FP16 decoding and rounding: numpy's float16 casts and CPython's struct 'e'
  codec (both independent, correctly rounded implementations).
- Packing: round trips, exhaustive code patterns, and the property the word
  layout is built for (a shift and a mask turn a word into FP16 pairs),
  checked through numpy's float16 view.
- Dequantisation: every one of the 65536 FP16 scale patterns times every
  code, against numpy's float16 product.
- GEMM: the closed form for all-ones activations (integer code sums times
  scales), exact rational arithmetic on tiny shapes, numpy's float64 matmul,
  and special cases (zero codes, zero scales, unit weights, sign symmetry).
- Storage: the effective-bit figures and size ratios the pages print.
"""
import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16)


def bits_equal_or_both_nan(a_bits, b_bits):
    a = np.asarray(a_bits, np.uint16)
    b = np.asarray(b_bits, np.uint16)
    an = np.isnan(f16(a))
    bn = np.isnan(f16(b))
    return np.where(an | bn, an & bn, a == b)


# --------------------------------------------------------------------- FP16
def test_half_decode_all_patterns(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle_mod.half_bits_to_double(bits)
    want = f16(bits).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def _rounding_candidates():
    pos = np.arange(0, 0x7C00, dtype=np.uint32).astype(np.uint16)  # all finite non-negative fp16
    v = f16(pos).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2  # exact in double
    top = np.array([65504.0, 65520.0])  # 65520: tie between 65504 and 2^16 (rounds to inf)
    mids = np.concatenate([mids, top[1:]])
    near = np.concatenate([np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)])
    rng = np.random.default_rng(7)
    logu = np.exp2(rng.uniform(-30, 17, 200_000)) * rng.choice([-1.0, 1.0], 200_000)
    uni = rng.uniform(-70000, 70000, 50_000)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 1e-300, -1e-300, 1e300, 2.0 ** -24, 2.0 ** -25,
                        3 * 2.0 ** -26, 2.0 ** -14, np.nextafter(2.0 ** -14, 0), 65519.999, 65520.0,
                        -65520.0, 1 + 2.0 ** -11 + 2.0 ** -40])
    return np.concatenate([v, -v, mids, -mids, near, -near, logu, uni, special])


def test_half_round_matches_numpy(oracle_mod):
    x = _rounding_candidates()
    got = oracle_mod.double_to_half_bits(x)
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_half_round_matches_struct_codec(oracle_mod):
    rng = np.random.default_rng(11)
    x = _rounding_candidates()
    x = x[np.abs(x) < 65520.0]  # struct refuses values that round to inf
    x = rng.choice(x, 20_000, replace=False)
    got = oracle_mod.double_to_half_bits(x)
    want = np.array([struct.unpack("<H", struct.pack("<e", float(v)))[0] for v in x], np.uint16)
    assert np.array_equal(got, want)


def test_half_round_nan(oracle_mod):
    got = oracle_mod.double_to_half_bits(np.array([np.nan, -np.nan]))
    assert np.all(np.isnan(f16(got)))


# ------------------------------------------------------------------ packing
@pytest.mark.parametrize("mode", ["binary", "ternary"])
@pytest.mark.parametrize("shape", [(1, 128), (3, 256), (17, 384), (64, 1024)])
def test_pack_round_trip(oracle_mod, mode, shape):
    rng = np.random.default_rng(shape[0] * 1000 + shape[1])
    c = workloads.codes(rng, shape[0], shape[1], mode)
    p = oracle_mod.pack(c, mode)
    assert p.dtype == np.uint32
    assert p.shape == (shape[0], shape[1] // (32 if mode == "binary" else 16))
    assert np.array_equal(oracle_mod.unpack(p, shape[1], mode), c)


def _ternary_pairs_as_fp16(words):
    """For each word and pair p: ((w << 2p) & 0xC000C000) read as two fp16."""
    w = np.asarray(words, np.uint32)
    out = []
    for p in range(8):
        x = (w << np.uint32(2 * p)) & np.uint32(0xC000C000)
        h = x.view(np.uint16).reshape(*w.shape, 2)  # little-endian: [..., 0] = low half
        out.append(f16(h).astype(np.float64))
    return np.stack(out, axis=-2).reshape(*w.shape[:-1], w.shape[-1] * 16)


def _binary_pairs_as_fp16(words):
    """For each word and pair p: (((w << p) & 0x80008000) | 0x3C003C00) read as two fp16."""
    w = np.asarray(words, np.uint32)
    out = []
    for p in range(16):
        x = ((w << np.uint32(p)) & np.uint32(0x80008000)) | np.uint32(0x3C003C00)
        h = x.view(np.uint16).reshape(*w.shape, 2)
        out.append(f16(h).astype(np.float64))
    return np.stack(out, axis=-2).reshape(*w.shape[:-1], w.shape[-1] * 32)


def test_ternary_layout_decodes_by_shift_and_mask(oracle_mod):
    """The INT2 layout is built so that one shift and one mask give the FP16
    pair (2*t[2p], 2*t[2p+1]); this checks it through numpy's fp16 view."""
    rng = np.random.default_rng(3)
    c = workloads.codes(rng, 40, 512, "ternary")
    p = oracle_mod.pack(c, "ternary")
    assert np.array_equal(_ternary_pairs_as_fp16(p), 2.0 * c)


def test_binary_layout_decodes_by_shift_and_mask(oracle_mod):
    rng = np.random.default_rng(4)
    c = workloads.codes(rng, 40, 512, "binary")
    p = oracle_mod.pack(c, "binary")
    assert np.array_equal(_binary_pairs_as_fp16(p), c.astype(np.float64))


def test_ternary_pack_exhaustive_patterns(oracle_mod):
    """All 3^8 patterns of the first and of the last 8 codes of a word."""
    grid = np.array(np.meshgrid(*[[-1, 0, 1]] * 8, indexing="ij")).reshape(8, -1).T.astype(np.int8)
    n = grid.shape[0]
    rng = np.random.default_rng(5)
    rest = workloads.codes(rng, n, 128, "ternary")
    for lo in (0, 8):
        c = rest.copy()
        c[:, lo:lo + 8] = grid
        p = oracle_mod.pack(c, "ternary")
        assert np.array_equal(oracle_mod.unpack(p, 128, "ternary"), c)
        assert np.array_equal(_ternary_pairs_as_fp16(p), 2.0 * c)
    assert len(np.unique(oracle_mod.pack(np.pad(grid, ((0, 0), (0, 120))), "ternary")[:, 0])) == n


def test_binary_pack_exhaustive_patterns(oracle_mod):
    """All 2^16 patterns of the first and of the last 16 codes of a word."""
    idx = np.arange(1 << 16, dtype=np.uint32)
    grid = np.where((idx[:, None] >> np.arange(16, dtype=np.uint32)) & 1, -1, 1).astype(np.int8)
    rng = np.random.default_rng(6)
    rest = workloads.codes(rng, grid.shape[0], 128, "binary")
    for lo in (0, 16):
        c = rest.copy()
        c[:, lo:lo + 16] = grid
        p = oracle_mod.pack(c, "binary")
        assert np.array_equal(oracle_mod.unpack(p, 128, "binary"), c)
        assert np.array_equal(_binary_pairs_as_fp16(p), c.astype(np.float64))


@pytest.mark.parametrize("mode,bad", [("ternary", 2), ("ternary", -2), ("ternary", 127), ("binary", 0),
                                      ("binary", 2), ("binary", -128)])
def test_pack_rejects_invalid_codes(oracle_mod, mode, bad):
    c = np.ones((4, 128), np.int8)
    c[2, 77] = bad
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.pack(c, mode)


def test_unpack_rejects_sign_without_magnitude(oracle_mod):
    p = np.zeros((1, 8), np.uint32)
    p[0, 3] = 1 << 15  # sign bit of weight 0 set, magnitude clear
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.unpack(p, 128, "ternary")


def test_pack_rejects_partial_group(oracle_mod):
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.pack(np.ones((2, 96), np.int8), "ternary")


# ----------------------------------------------------------------- dequant
@pytest.mark.parametrize("mode", ["binary", "ternary"])
def test_dequant_every_scale_pattern(oracle_mod, mode):
    """w = t*s for all 65536 fp16 scale patterns and every code, against
    numpy's float16 product (NaN results compared as NaN)."""
    K = 128
    s_bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rng = np.random.default_rng(8)
    c = workloads.codes(rng, 65536, K, mode)
    c[:, :3] = [-1, 1, -1] if mode == "binary" else [-1, 0, 1]  # every code in every row
    p = oracle_mod.pack(c, mode)
    w = oracle_mod.dequant(p, s_bits[:, None], K, mode)
    with np.errstate(invalid="ignore", over="ignore"):
        want = (c.astype(np.float16) * f16(s_bits)[:, None]).view(np.uint16)
    assert np.all(bits_equal_or_both_nan(w, want))


def test_dequant_values_are_plus_minus_scale_or_zero(oracle_mod):
    d = workloads.make(workloads.TERNARY_TINY)
    p = oracle_mod.pack(d["codes"], "ternary")
    w = oracle_mod.dequant(p, d["scales"], d["K"], "ternary").astype(np.uint32)
    s = np.repeat(d["scales"], 128, axis=1).astype(np.uint32)
    c = d["codes"]
    assert np.array_equal(w[c == 1], s[c == 1])
    assert np.array_equal(w[c == -1], s[c == -1] ^ 0x8000)
    assert np.all(w[c == 0] == 0)  # positive scales: +0


# -------------------------------------------------------------------- GEMM
def _ones_closed_form(codes, scales_bits, K):
    """out[n] = sum_g s_g * sum_{k in g} t[n,k]: integer code sums per group
    times the scale, added in Python floats (exact here)."""
    N = codes.shape[0]
    G = K // 128
    tsum = codes.reshape(N, G, 128).astype(np.int64).sum(axis=2)
    s = f16(scales_bits).astype(np.float64)
    out = np.zeros(N)
    for n in range(N):
        out[n] = math.fsum(float(s[n, g]) * int(tsum[n, g]) for g in range(G))
    return out


@pytest.mark.parametrize("mode", ["binary", "ternary"])
@pytest.mark.parametrize("N,K", [(16, 128), (33, 384), (64, 1024)])
def test_gemm_all_ones_closed_form(oracle_mod, mode, N, K):
    rng = np.random.default_rng(N + K)
    c = workloads.codes(rng, N, K, mode)
    s = rng.uniform(-0.3, 0.3, (N, K // 128)).astype(np.float16).view(np.uint16)  # both signs
    A = np.full((3, K), np.float16(1.0)).view(np.uint16)
    p = oracle_mod.pack(c, mode)
    out, acc, absacc = oracle_mod.gemm(A, p, s, K, mode, threads=2)
    want = _ones_closed_form(c, s, K)
    for m in range(3):
        assert np.array_equal(acc[m], want)
    assert np.array_equal(out[0], oracle_mod.double_to_half_bits(want))


@pytest.mark.parametrize("mode", ["binary", "ternary"])
@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (2, 3, 128), (4, 16, 256), (3, 5, 384)])
def test_gemm_brute_force_exact_rationals(oracle_mod, mode, M, N, K):
    """Tiny shapes against a triple loop in exact rational arithmetic written
    here from the definition out[m,n] = sum_k A[m,k] * t[n,k] * s[n, k//128]."""
    d = workloads.make(mode=mode, M=M, N=N, K=K, seed=M * 100 + N * 10 + K)
    p = oracle_mod.pack(d["codes"], mode)
    out, acc, absacc = oracle_mod.gemm(d["A"], p, d["scales"], K, mode, threads=1)
    a = [[Fraction(float(v)) for v in row] for row in f16(d["A"])]
    s = [[Fraction(float(v)) for v in row] for row in f16(d["scales"])]
    t = d["codes"].tolist()
    for m in range(M):
        for n in range(N):
            exact = sum(a[m][k] * t[n][k] * s[n][k // 128] for k in range(K))
            mag = sum(abs(a[m][k] * t[n][k] * s[n][k // 128]) for k in range(K))
            assert abs(Fraction(acc[m, n]) - exact) <= Fraction(K, 2 ** 53) * mag
            assert Fraction(absacc[m, n]) == mag or abs(Fraction(absacc[m, n]) - mag) <= Fraction(K, 2 ** 53) * mag


@pytest.mark.parametrize("mode", ["binary", "ternary"])
def test_gemm_matches_numpy_matmul(oracle_mod, mode):
    d = workloads.make(mode=mode, M=37, N=70, K=640, seed=21)
    p = oracle_mod.pack(d["codes"], mode)
    out, acc, absacc = oracle_mod.gemm(d["A"], p, d["scales"], 640, mode)
    W = d["codes"].astype(np.float64) * np.repeat(f16(d["scales"]).astype(np.float64), 128, axis=1)
    ref = f16(d["A"]).astype(np.float64) @ W.T
    assert np.allclose(acc, ref, rtol=0, atol=1e-12 * np.abs(W).sum(axis=1).max() * 8)
    assert np.allclose(absacc, np.abs(f16(d["A"]).astype(np.float64)) @ np.abs(W).T, rtol=1e-13)


def test_gemm_special_cases(oracle_mod):
    rng = np.random.default_rng(9)
    K = 256
    A = workloads.activations(rng, 5, K)
    # zero codes -> +0 everywhere
    z = np.zeros((8, K), np.int8)
    s = workloads.scales(rng, 8, K)
    out, acc, _ = oracle_mod.gemm(A, oracle_mod.pack(z, "ternary"), s, K, "ternary")
    assert np.all(out == 0) and np.all(acc == 0)
    # zero scales -> zeros
    c = workloads.codes(rng, 8, K, "binary")
    out, acc, _ = oracle_mod.gemm(A, oracle_mod.pack(c, "binary"), np.zeros((8, 2), np.uint16), K, "binary")
    assert np.all(acc == 0)
    # all +1 codes with unit scales -> exact row sums of A
    one = np.full((4, K // 128), np.float16(1.0)).view(np.uint16)
    out, acc, _ = oracle_mod.gemm(A, oracle_mod.pack(np.ones((4, K), np.int8), "binary"), one, K, "binary")
    rows = [math.fsum(float(v) for v in r) for r in f16(A)]
    for m in range(5):
        assert np.all(acc[m] == rows[m])


@pytest.mark.parametrize("mode", ["binary", "ternary"])
def test_gemm_sign_and_power_of_two_symmetry(oracle_mod, mode):
    d = workloads.make(mode=mode, M=9, N=24, K=384, seed=31)
    p = oracle_mod.pack(d["codes"], mode)
    pn = oracle_mod.pack(-d["codes"], mode)
    out, acc, _ = oracle_mod.gemm(d["A"], p, d["scales"], 384, mode)
    out_n, acc_n, _ = oracle_mod.gemm(d["A"], pn, d["scales"], 384, mode)
    assert np.array_equal(acc_n, -acc)
    nz = acc != 0
    assert np.array_equal(out_n[nz], out[nz] ^ np.uint16(0x8000))
    A2 = (f16(d["A"]).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    _, acc2, _ = oracle_mod.gemm(A2, p, d["scales"], 384, mode)
    assert np.array_equal(acc2, 2 * acc)


def test_gemm_entries_and_thread_count(oracle_mod):
    d = workloads.make(mode="ternary", M=23, N=41, K=256, seed=41)
    p = oracle_mod.pack(d["codes"], "ternary")
    out1, acc1, abs1 = oracle_mod.gemm(d["A"], p, d["scales"], 256, "ternary", threads=1)
    out4, acc4, abs4 = oracle_mod.gemm(d["A"], p, d["scales"], 256, "ternary", threads=4)
    assert np.array_equal(acc1, acc4) and np.array_equal(out1, out4)
    ms = np.array([0, 22, 5, 11])
    ns = np.array([0, 40, 17, 3])
    o, a, b = oracle_mod.gemm_entries(d["A"], p, d["scales"], 256, "ternary", ms, ns)
    assert np.array_equal(o, out1[ms, ns]) and np.array_equal(a, acc1[ms, ns]) and np.array_equal(b, abs1[ms, ns])


def test_tolerance_helper(oracle_mod):
    ref = np.float16([1.0, 1000.0, 0.0, np.inf]).view(np.uint16)
    gpu_ok = np.float16([1.0009765625, 1000.5, 2.0 ** -24, np.inf]).view(np.uint16)
    gpu_bad = np.float16([1.5, 1003.0, 0.01, 65504.0]).view(np.uint16)
    absacc = np.array([0.0, 1.0, 0.0, 1.0])
    assert oracle_mod.within_tolerance(gpu_ok, ref, absacc).all()
    assert not oracle_mod.within_tolerance(gpu_bad, ref, absacc).any()


# ----------------------------------------------------------------- storage
def _golden():
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        return json.load(f)


def test_effective_bits_match_pages(oracle_mod):
    g = _golden()
    N, K = 3072, 9216
    gs = g["group_size"]["value"]
    sb = g["scale_bits"]["value"]
    scale_bytes = N * (K // gs) * sb // 8
    bits_bin = 8 * (oracle_mod.packed_bytes(N, K, "binary") + scale_bytes) / (N * K)
    assert bits_bin == g["binary_effective_bits"]["value"]  # 1 + 16/128 exactly
    bits_int2 = 8 * (oracle_mod.packed_bytes(N, K, "ternary") + scale_bytes) / (N * K)
    assert bits_int2 == g["int2_bits_per_ternary_weight"]["value"] + sb / gs  # 2.125
    info = math.log2(3)
    assert round(info, 3) == g["ternary_information_bits"]["value"]
    assert round(info + sb / gs, 2) == g["ternary_effective_bits"]["value"]
    assert round(16 / bits_bin) == g["binary_layer_reduction"]["value"]
    assert round(16 / g["ternary_effective_bits"]["value"], 1) == g["ternary_layer_reduction"]["value"]


def test_page_sizes_are_consistent():
    """The 0.93 / 1.21 GB transformers at 1.125 / 1.71 bits imply one count of
    quantised weights and an FP16 remainder near the stated ~5%."""
    g = _golden()
    tb = g["transformer_gb"]
    x = (tb["ternary"] - tb["binary"]) * 1e9 * 8 / (g["ternary_effective_bits"]["value"] - 1.125)
    fp16_bytes = tb["binary"] * 1e9 - x * 1.125 / 8
    fp16_params = fp16_bytes / 2
    frac = fp16_params / (x + fp16_params)
    assert 3.5e9 < x < 4.2e9
    assert 0.02 < frac < 0.08
    assert round(tb["full_precision"] / tb["binary"], 1) == g["transformer_reduction"]["binary"]
    assert round(tb["full_precision"] / tb["ternary"], 1) == g["transformer_reduction"]["ternary"]


def test_stack_layer_lists():
    """80 launches with Q|K|V stacked and 100 with them split cover the same
    weights: 2,831,155,200 for a hidden-3072, 25-block MMDiT."""
    fused = workloads.mmdit_stack_layers()
    split = workloads.mmdit_stack_layers(split_qkv=True)
    assert len(fused) == 80 and len(split) == 100
    total = sum(n * k for _, n, k in fused)
    assert total == sum(n * k for _, n, k in split) == 2_831_155_200


def test_stream_layer_lists():
    """With real per-stream token counts each double-stream block has its
    image and text linears on their own rows and the single-stream blocks run
    on the joint sequence; the weights are the same 2,831,155,200."""
    layers = workloads.mmdit_stream_layers(4096, 512)
    assert len(layers) == 80
    assert sum(n * k for _, _, n, k in layers) == 2_831_155_200
    rows = {}
    for name, m, _, _ in layers:
        kind = "single" if name.startswith("single") else ("img" if ".img." in name else "txt")
        rows.setdefault(kind, set()).add(m)
    assert rows == {"img": {4096}, "txt": {512}, "single": {4608}}
    # 5 blocks x (4 image + 4 text linears) + 20 x 2 single-stream ones
    assert sum(1 for name, *_ in layers if ".img." in name) == 20
    assert sum(1 for name, *_ in layers if ".txt." in name) == 20


# ------------------------------------------------ base-3 ternary format --
# This project's denser format (five trits per byte; not on the pages, which
# only state the 1.71-bit information figure and 2-bit INT2 storage): byte j
# of a 128-weight group holds the weights at positions j, j+26, j+52, j+78,
# j+104 as the base-3 digits of v = sum (t+1) 3^(4-i), most significant
# first, stored as ceil(256 v / 243); 26 bytes per group, four groups per
# 112-byte block (8 zero bytes at its end), blocks along the row.


def _b3_byte(v):
    """ceil(256 v / 243), exactly, in rational arithmetic."""
    return math.ceil(Fraction(256 * v, 243))

def _b3_digits_lsb_first(b):
    """Base-3 digits of b, least significant first, by repeated division."""
    out = []
    for _ in range(5):
        b, r = divmod(b, 3)
        out.append(r)
    return out


def test_b3_every_byte_value_at_every_position(oracle_mod):
    """Exhaustive: each of the 243 byte values at each of the 26 byte
    positions decodes to its base-3 digits at positions j + 26 i (digit i
    counted from the most significant), zero bytes around it to t = -1."""
    K = 128
    zero = _b3_byte(0)
    assert zero == 0  # all-zero padding bytes are valid (v = 0)
    for j in range(26):
        rows = []
        expected = []
        for v in range(243):
            d = _b3_digits_lsb_first(v)[::-1]  # most significant first
            if j >= 24 and d[4] != 0:
                continue  # the last digit of bytes 24, 25 is padding and must be zero
            row = np.zeros(112, np.uint8)
            row[j] = _b3_byte(v)
            rows.append(row)
            t = np.full(K, -1, np.int8)
            for i in range(5):
                if 26 * i + j < K:
                    t[26 * i + j] = d[i] - 1
            expected.append(t)
        packed = np.stack(rows).view(np.uint32)
        got = oracle_mod.unpack(packed, K, "ternary_b3")
        assert np.array_equal(got, np.stack(expected)), j


def test_b3_rejects_what_is_not_a_code(oracle_mod):
    good = oracle_mod.pack(np.zeros((1, 128), np.int8), "ternary_b3")
    valid = {_b3_byte(v) for v in range(243)}
    assert len(valid) == 243
    not_codes = sorted(set(range(256)) - valid)
    assert len(not_codes) == 13
    # bytes that are no code; a padding digit; an unused group slot; block padding
    cases = [(3, b) for b in not_codes] + [(24, _b3_byte(1)), (25, _b3_byte(2)), (26, 1), (31, 7), (104, 1),
                                            (111, 255)]
    for pos, value in cases:
        bad = good.copy().view(np.uint8)
        bad[0, pos] = value  # a byte above 242, a padding digit, row padding
        with pytest.raises(oracle_mod.OracleError):
            oracle_mod.unpack(bad.view(np.uint32), 128, "ternary_b3")
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.pack(np.full((1, 128), 2, np.int8), "ternary_b3")


@pytest.mark.parametrize("K", [128, 256, 384, 1024, 3072])
def test_b3_round_trip_and_size(oracle_mod, K):
    rng = np.random.default_rng(K)
    N = 7
    codes = workloads.codes(rng, N, K, "ternary")
    packed = oracle_mod.pack(codes, "ternary_b3")
    assert np.array_equal(oracle_mod.unpack(packed, K, "ternary_b3"), codes)
    row = 112 * -(-(K // 128) // 4)
    assert oracle_mod.packed_bytes(N, K, "ternary_b3") == N * row == packed.nbytes
    # 112 bytes per 512 weights: 1.75 bits (1.625 of them trits), above
    # log2(3) = 1.585 and below the 2 bits of INT2; with the FP16 scale per
    # group 1.875 bits per weight against INT2's 2.125.
    assert 112 * 8 / 512 == 1.75 and 26 * 8 / 128 == 1.625
    assert np.log2(3) < 1.625 < 1.75 < 2.0
    assert (112 * 8 + 4 * 16) / 512 == 1.875


def test_b3_row_layout(oracle_mod):
    """A row of 5 groups (two blocks) built by concatenation: per block the
    26-byte groups in order, then zero bytes up to 112."""
    rng = np.random.default_rng(5)
    K = 640
    codes = workloads.codes(rng, 3, K, "ternary")
    for n in range(3):
        groups = []
        for g in range(K // 128):
            t = codes[n, 128 * g:128 * (g + 1)].astype(int)
            q = list(t + 1) + [0, 0]  # two padding positions, digit 0
            groups.append(bytes(_b3_byte(sum(q[26 * i + j] * 3 ** (4 - i) for i in range(5))) for j in range(26)))
        blocks = [b"".join(groups[b:b + 4]) for b in range(0, len(groups), 4)]
        expected = b"".join(blk + bytes(112 - len(blk)) for blk in blocks)
        got = oracle_mod.pack(codes, "ternary_b3")[n].tobytes()
        assert got == expected, n


def test_b3_weights_and_gemm_equal_int2_on_the_same_codes(oracle_mod):
    """Same codes, two storage formats: the dequantised weights and the GEMM
    (outputs, double sums, absolute sums) are identical."""
    d = workloads.make(mode="ternary", M=9, N=33, K=640, seed=51)
    p2 = oracle_mod.pack(d["codes"], "ternary")
    p3 = oracle_mod.pack(d["codes"], "ternary_b3")
    assert np.array_equal(oracle_mod.dequant(p2, d["scales"], 640, "ternary"),
                          oracle_mod.dequant(p3, d["scales"], 640, "ternary_b3"))
    o2, a2, s2 = oracle_mod.gemm(d["A"], p2, d["scales"], 640, "ternary")
    o3, a3, s3 = oracle_mod.gemm(d["A"], p3, d["scales"], 640, "ternary_b3")
    assert np.array_equal(o2, o3) and np.array_equal(a2, a3) and np.array_equal(s2, s3)
    ms, ns = np.array([0, 8, 4]), np.array([32, 0, 17])
    e3 = oracle_mod.gemm_entries(d["A"], p3, d["scales"], 640, "ternary_b3", ms, ns)
    assert np.array_equal(e3[0], o2[ms, ns]) and np.array_equal(e3[1], a2[ms, ns])


# ------------------------------------------- 4-bit group-affine weights --
# The pages name "4-bit HQQ" for the text encoder and nothing more; the
# oracle reads it as HQQ's scheme w = fp16(fp16(q - z) * s), groups of 64
# along K, with this project's packing.  What is pinned below is that
# reading's arithmetic and layout; the reading itself is unpinned.

def test_hqq4_layout_shift_and_mask(oracle_mod):
    """Weights 2p, 2p+1 of a word come out of (word >> 4p) & 0x000F000F as
    the low and high 16-bit halves, for every nibble value in every slot."""
    rng = np.random.default_rng(3)
    q = rng.integers(0, 16, (64, 256)).astype(np.uint8)
    q[0, :16] = np.arange(16)
    words = oracle_mod.hqq4_pack(q).astype(np.uint64)
    for p in range(4):
        pair = (words >> np.uint64(4 * p)) & np.uint64(0x000F000F)
        assert np.array_equal(pair & np.uint64(0xFFFF), q[:, 2 * p::8].astype(np.uint64))
        assert np.array_equal(pair >> np.uint64(16), q[:, 2 * p + 1::8].astype(np.uint64))
    assert np.array_equal(oracle_mod.hqq4_unpack(oracle_mod.hqq4_pack(q), 256), q)
    bad = q.copy()
    bad[5, 7] = 16
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.hqq4_pack(bad)


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16)


def test_hqq4_dequant_matches_ieee_fp16_arithmetic(oracle_mod):
    """w = fp16(fp16(q - z) * s) against numpy's float16 operations (each an
    exactly computed result rounded once): every scale pattern with random q
    and zero, and zeros / scales at the special values."""
    rng = np.random.default_rng(11)
    N, K = 1024, 128
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    scales = np.arange(N * 2, dtype=np.uint32).astype(np.uint16).reshape(N, 2)  # 2048 of the patterns
    scales[:, 1] = rng.integers(0, 65536, N).astype(np.uint16)
    zeros = rng.integers(0, 65536, (N, 2)).astype(np.uint16)
    specials = np.array([0x0000, 0x8000, 0x3C00, 0x4700, 0x4B80, 0x7C00, 0xFC00, 0x7E00, 0x0001, 0x03FF],
                        np.uint16)
    zeros[:len(specials), 0] = specials
    scales[len(specials):2 * len(specials), 0] = specials
    got = oracle_mod.hqq4_dequant(oracle_mod.hqq4_pack(q), scales, zeros, K)
    with np.errstate(all="ignore"):
        zz = np.repeat(_f16(zeros), 64, axis=1)
        ss = np.repeat(_f16(scales), 64, axis=1)
        want = ((q.astype(np.float16) - zz).astype(np.float16) * ss).astype(np.float16)
    assert np.all(nan_equal(got, want.view(np.uint16)))
    for start in range(0, 65536, 8192):  # every scale pattern once, with q and z varying
        s_all = (np.arange(start, start + 8192, dtype=np.uint32).astype(np.uint16)).reshape(-1, 2)
        z_all = rng.integers(0, 65536, s_all.shape).astype(np.uint16)
        q_all = rng.integers(0, 16, (s_all.shape[0], 128)).astype(np.uint8)
        got = oracle_mod.hqq4_dequant(oracle_mod.hqq4_pack(q_all), s_all, z_all, 128)
        with np.errstate(all="ignore"):
            want = ((q_all.astype(np.float16) - np.repeat(_f16(z_all), 64, axis=1)).astype(np.float16) *
                    np.repeat(_f16(s_all), 64, axis=1)).astype(np.float16)
        assert np.all(nan_equal(got, want.view(np.uint16)))


def nan_equal(a, b):
    a = np.asarray(a, np.uint16)
    b = np.asarray(b, np.uint16)
    an, bn = np.isnan(a.view(np.float16)), np.isnan(b.view(np.float16))
    return np.where(an | bn, an & bn, a == b)


def test_hqq4_gemm_all_ones_closed_form(oracle_mod):
    """With all-ones activations every output's double sum is exactly the sum
    of the row's FP16 weights (each a multiple of 2^-24 below 2^16, so the
    sums are exact in double)."""
    rng = np.random.default_rng(13)
    N, K = 40, 512
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    scales = np.float16(rng.uniform(0.001, 0.1, (N, K // 64))).view(np.uint16)
    zeros = np.float16(rng.uniform(0.0, 15.0, (N, K // 64))).view(np.uint16)
    packed = oracle_mod.hqq4_pack(q)
    w = ((q.astype(np.float16) - np.repeat(_f16(zeros), 64, axis=1)).astype(np.float16) *
         np.repeat(_f16(scales), 64, axis=1)).astype(np.float16)
    want = w.astype(np.float64).sum(axis=1)
    A = np.full((3, K), 0x3C00, np.uint16)  # 1.0
    out, acc, absacc = oracle_mod.hqq4_gemm(A, packed, scales, zeros, K)
    assert np.array_equal(acc, np.broadcast_to(want, acc.shape))
    assert np.array_equal(absacc, np.broadcast_to(np.abs(w.astype(np.float64)).sum(axis=1), acc.shape))
    assert np.array_equal(out, oracle_mod.double_to_half_bits(acc))
