"""GPU parity: the CUDA library, called through its C ABI, against the CPU
oracle on the same seeded inputs.

Bars: pack and dequant bit-exact (NaN compared as NaN); GEMM element-wise
|gpu - oracle| <= 1e-3 * sum_k |a_k w_k| + one FP16 ulp of the oracle value.
Small and ragged shapes are compared in full; the full-size workloads at the
positions the oracle computes one by one (random positions plus every tile
edge and the last row and column).
"""
import numpy as np
import pytest
import torch

import bit_weight_gemm_b200 as bw
import workloads

pytestmark = pytest.mark.gpu

RTOL = 1e-3
MODES = ["binary", "ternary", "ternary_b3"]  # ternary_b3: the same codes in the base-3 storage format


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    bw.lib()
    assert bw.get_device_error() == 0
    yield
    assert bw.get_device_error() == 0, "a kernel recorded a device-side error"


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def to_u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_u32(t):
    return t.cpu().contiguous().numpy().view(np.uint32)


def nan_aware_equal(a, b):
    a = np.asarray(a, np.uint16)
    b = np.asarray(b, np.uint16)
    an = np.isnan(a.view(np.float16))
    bn = np.isnan(b.view(np.float16))
    return np.where(an | bn, an & bn, a == b)


def gpu_inputs(d, oracle_mod):
    packed_ref = oracle_mod.pack(d["codes"], d["mode"])
    codes = dev(d["codes"])
    packed = bw.pack(codes, d["mode"])
    torch.cuda.synchronize()
    return packed_ref, packed, dev(d["A"].view(np.int16), torch.float16), dev(d["scales"].view(np.int16), torch.float16)


def assert_gemm_close(oracle_mod, got_bits, ref_bits, absacc, label):
    ok = oracle_mod.within_tolerance(got_bits, ref_bits, absacc, RTOL)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        g = oracle_mod.half_bits_to_double(got_bits)
        r = oracle_mod.half_bits_to_double(ref_bits)
        details = [(tuple(i), g[tuple(i)], r[tuple(i)], absacc[tuple(i)]) for i in idx]
        pytest.fail(f"{label}: {int((~ok).sum())} of {ok.size} outside tolerance, e.g. {details}")


# ------------------------------------------------------------------ pack
PACK_SHAPES = [(1, 128), (37, 384), (256, 256), (129, 1152), (1000, 3072)]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("N,K", PACK_SHAPES)
def test_pack_bit_exact(oracle_mod, mode, N, K):
    d = workloads.make(mode=mode, M=1, N=N, K=K, seed=N * 7 + K)
    ref = oracle_mod.pack(d["codes"], mode)
    got = bw.pack(dev(d["codes"]), mode)
    assert np.array_equal(to_u32(got), ref)


@pytest.mark.parametrize("mode", MODES)
def test_pack_bit_exact_from_16_byte_aligned_codes(oracle_mod, mode):
    """Codes that are 16- but not 32-byte aligned take the 16-byte load path."""
    d = workloads.make(mode=mode, M=1, N=129, K=1152, seed=99)
    buf = torch.empty(d["codes"].size + 16, dtype=torch.int8, device="cuda")
    assert buf.data_ptr() % 32 == 0
    codes = buf[16:].view(129, 1152)
    codes.copy_(dev(d["codes"]))
    assert codes.data_ptr() % 32 == 16
    assert np.array_equal(to_u32(bw.pack(codes, mode)), oracle_mod.pack(d["codes"], mode))


@pytest.mark.parametrize("mode,bad", [("ternary", 2), ("ternary", -2), ("binary", 0), ("binary", 3),
                                      ("ternary_b3", 2), ("ternary_b3", -128)])
def test_pack_reports_bad_codes(mode, bad):
    c = np.ones((64, 256), np.int8)
    c[63, 255] = bad
    with pytest.raises(bw.BonsaiError) as e:
        bw.pack(dev(c), mode)
    assert e.value.status == 4
    c[63, 255] = 1
    bw.pack(dev(c), mode)  # the flag was reset by the failing call


# --------------------------------------------------------------- dequant
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("N,K", PACK_SHAPES)
def test_dequant_bit_exact(oracle_mod, mode, N, K):
    d = workloads.make(mode=mode, M=1, N=N, K=K, seed=N * 3 + K)
    ref_packed, packed, _, scales = gpu_inputs(d, oracle_mod)
    ref = oracle_mod.dequant(ref_packed, d["scales"], K, mode)
    got = bw.dequant(packed, scales, K, mode)
    assert np.all(nan_aware_equal(to_u16(got), ref))


@pytest.mark.parametrize("mode", MODES)
def test_dequant_bit_exact_into_16_byte_aligned_output(oracle_mod, mode):
    """An output 16- but not 32-byte aligned takes the 16-byte store path."""
    N, K = 129, 1152
    d = workloads.make(mode=mode, M=1, N=N, K=K, seed=98)
    ref_packed, packed, _, scales = gpu_inputs(d, oracle_mod)
    buf = torch.empty(N * K + 8, dtype=torch.float16, device="cuda")
    assert buf.data_ptr() % 32 == 0
    out = buf[8:].view(N, K)
    assert out.data_ptr() % 32 == 16
    bw.dequant(packed, scales, K, mode, out=out)
    assert np.all(nan_aware_equal(to_u16(out), oracle_mod.dequant(ref_packed, d["scales"], K, mode)))


@pytest.mark.parametrize("mode", MODES)
def test_dequant_every_scale_pattern(oracle_mod, mode):
    N, K = 65536, 128
    rng = np.random.default_rng(12)
    c = workloads.codes(rng, N, K, mode)
    s = np.arange(N, dtype=np.uint32).astype(np.uint16)[:, None]
    ref_packed = oracle_mod.pack(c, mode)
    ref = oracle_mod.dequant(ref_packed, s, K, mode)
    got = bw.dequant(dev(ref_packed.view(np.int32)), dev(s.view(np.int16), torch.float16), K, mode)
    assert np.all(nan_aware_equal(to_u16(got), ref))


# ------------------------------------------------------------------ GEMM
SMALL_SHAPES = [
    (1, 8, 128), (5, 130, 256), (16, 128, 128), (17, 200, 384), (33, 256, 640), (64, 384, 256),
    (65, 129, 1152), (128, 256, 512), (129, 300, 256), (255, 128, 384), (256, 512, 256), (300, 384, 512),
    (513, 136, 768),
    # few tiles, many groups: K is split over a cluster (sizes 2..8, not only powers of two)
    (16, 256, 4096), (40, 384, 2048), (7, 128, 640), (100, 264, 1152), (16, 3072, 1024),
]


def _gemm_case(oracle_mod, mode, M, N, K, seed):
    d = workloads.make(mode=mode, M=M, N=N, K=K, seed=seed)
    ref_packed, packed, A, scales = gpu_inputs(d, oracle_mod)
    out = bw.lowbit_gemm(A, packed, scales, mode)
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.gemm(d["A"], ref_packed, d["scales"], K, mode)
    return to_u16(out), ref, absacc


def test_gemm_ternary_tiny_config(oracle_mod):
    p = workloads.TERNARY_TINY
    got, ref, absacc = _gemm_case(oracle_mod, p.mode, p.M, p.N, p.K, p.seed)
    assert_gemm_close(oracle_mod, got, ref, absacc, p.name)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,N,K", SMALL_SHAPES)
def test_gemm_ragged_shapes(oracle_mod, mode, M, N, K):
    got, ref, absacc = _gemm_case(oracle_mod, mode, M, N, K, seed=M * 31 + N * 7 + K)
    assert_gemm_close(oracle_mod, got, ref, absacc, f"{mode} {M}x{N}x{K}")


def test_gemm_binary_512_linear_full(oracle_mod):
    p = workloads.BINARY_512_LINEAR
    got, ref, absacc = _gemm_case(oracle_mod, p.mode, p.M, p.N, p.K, p.seed)
    assert_gemm_close(oracle_mod, got, ref, absacc, p.name)


def _sample_positions(M, N, block_t, count, seed):
    rng = np.random.default_rng(seed)
    ms = list(rng.integers(0, M, count))
    ns = list(rng.integers(0, N, count))
    edges_m = sorted({0, M - 1} | {x for b in range(block_t, M, block_t) for x in (b - 1, b)})
    edges_n = sorted({0, N - 1} | {x for b in range(128, N, 128) for x in (b - 1, b)})
    for m in edges_m[:64]:
        ms += [m] * 8
        ns += list(rng.integers(0, N, 8))
    for n in edges_n[:160]:
        ms += list(rng.integers(0, M, 4))
        ns += [n] * 4
    return np.array(ms, np.int64), np.array(ns, np.int64)


FULL = [workloads.TERNARY_MLP_UP_4608, workloads.TERNARY_MLP_DOWN_4608, workloads.TERNARY_QKV_4608,
        workloads.TERNARY_MLP_DOWN_16, workloads.TERNARY_QKV_16,
        workloads.Problem("base-3 ternary MLP-up M=4608", "ternary_b3", 4608, 9216, 3072, 1003),
        workloads.Problem("base-3 ternary MLP-down M=16", "ternary_b3", 16, 3072, 9216, 1014)]


@pytest.mark.parametrize("problem", FULL, ids=[p.name for p in FULL])
def test_gemm_full_size_sampled(oracle_mod, problem):
    d = workloads.make(problem)
    ref_packed, packed, A, scales = gpu_inputs(d, oracle_mod)
    out = bw.lowbit_gemm(A, packed, scales, problem.mode)
    got = to_u16(out)
    ms, ns = _sample_positions(problem.M, problem.N, 256 if problem.M > 128 else 16, 3000, problem.seed)
    ref, _, absacc = oracle_mod.gemm_entries(d["A"], ref_packed, d["scales"], problem.K, problem.mode, ms, ns)
    assert_gemm_close(oracle_mod, got[ms, ns], ref, absacc, problem.name)
    # every output written: no NaN/inf (inputs are bounded) and no untouched rows
    assert np.isfinite(got.view(np.float16)).all()


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def test_plans_cover_every_form():
    big = bw.gemm_plan(4608, 9216, 3072, "ternary")  # persistent: one CTA per SM walks 1296 tiles
    assert big == {"block_t": 256, "ksplit": 1, "ctas": _sms(), "tiles": 72 * 18}
    one_wave = bw.gemm_plan(1024, 3072, 3072, "binary")  # 144 176-token tiles: one CTA each, one wave
    assert one_wave["block_t"] == 176 and one_wave["tiles"] == 24 * 6
    assert one_wave["ctas"] == one_wave["tiles"] * one_wave["ksplit"]
    for M, N, K in [(16, 3072, 9216), (16, 256, 4096), (40, 384, 2048)]:
        p = bw.gemm_plan(M, N, K, "ternary")
        assert 1 < p["ksplit"] <= 8 and p["ctas"] == p["tiles"] * p["ksplit"], (M, N, K, p)
    # 72 tiles of 24 groups at 16 tokens: no split, on half the SMs (the next launch starts beside it)
    assert bw.gemm_plan(16, 9216, 3072, "ternary") == {"block_t": 16, "ksplit": 1, "ctas": 72, "tiles": 72}
    assert bw.gemm_plan(0, 8, 128, "binary") == {"block_t": 0, "ksplit": 0, "ctas": 0, "tiles": 0}


def test_plan_in_a_fresh_process_matches_launch():
    """The plan query before any launch in the process (occupancy of the
    split-K clusters depends on the kernels' shared-memory opt-in) gives the
    plan a launch uses."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import json, bit_weight_gemm_b200 as bw; "
            "print(json.dumps([bw.gemm_plan(16, 3072, 9216, 'ternary'), bw.gemm_plan(40, 384, 2048, 'binary')]))")
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    fresh = json.loads(res.stdout.strip().splitlines()[-1])
    assert fresh[0]["ksplit"] > 1 and fresh[1]["ksplit"] > 1, fresh
    assert fresh == [bw.gemm_plan(16, 3072, 9216, "ternary"), bw.gemm_plan(40, 384, 2048, "binary")]


# Large M: more tiles than SMs.  With K a multiple of 512 (ternary) or 1024
# (binary) one persistent CTA per SM walks the 256-token tiles; else each
# 128- or 256-token tile is its own CTA over several waves.  Ragged M and N;
# 234, 225 and 237 tiles leave persistent CTAs with one and with two tiles;
# N odd in the fifth case.  (N is wide enough that 352-token tiles would not
# fit one wave, so these shapes keep the forms they test.)
LARGE_M_SHAPES = [
    ("ternary", 1357, 4990, 512, True),
    ("ternary_b3", 1357, 4990, 512, True),
    ("ternary_b3", 700, 9600, 1152, False),
    ("binary", 700, 9600, 1024, True),
    ("ternary", 513, 9999, 1024, True),
    ("ternary", 1357, 4990, 640, False),
    ("binary", 600, 9600, 512, False),
]


# Mid-M token tiles, where 256-token ones would leave SMs idle: one wave of
# one-tile CTAs of 176 tokens (M=1024 / 1000 with N=3072 / 3000: 144 tiles)
# and the persistent kernel with 192-token tiles (M=2048 with N=3072: 264
# tiles); ragged M and N, in every format (the 4-bit weights at 1000 x 3000
# in test_hqq4_gemm_full).
MID_M_TILE_SHAPES = [
    ("binary", 1024, 3072, 3072, 176, False),
    ("ternary", 1000, 3000, 1152, 176, False),
    ("ternary_b3", 1000, 3000, 1152, 176, False),
    ("ternary", 1024, 3072, 12288, 176, False),
    ("ternary", 2304, 3072, 2048, 192, True),
    ("ternary_b3", 2300, 3050, 2048, 192, True),
    ("binary", 2304, 3072, 2048, 192, True),
    # 352-token tiles (two 176-token halves, ternary formats): 144 one-wave CTAs at ~2048 tokens on N ~ 3072
    ("ternary", 2048, 3072, 2048, 352, False),
    ("ternary_b3", 2000, 3050, 2048, 352, False),
    ("ternary", 1800, 3072, 2048, 352, False),  # the last tile's second half starts past M: not stored
    ("ternary", 2048, 2996, 1152, 352, False),  # N % 8 != 0: direct stores instead of TMA
    ("ternary_b3", 700, 6376, 1152, 352, False),  # 100 tiles, where 256-token ones make 150 (two waves)
]


@pytest.mark.parametrize("mode,M,N,K,block_t,persistent", MID_M_TILE_SHAPES)
def test_gemm_mid_m_token_tiles(oracle_mod, mode, M, N, K, block_t, persistent):
    plan = bw.gemm_plan(M, N, K, mode)
    assert plan["block_t"] == block_t and plan["ksplit"] == 1, plan
    assert (plan["ctas"] < plan["tiles"]) == persistent, plan
    got, ref, absacc = _gemm_case(oracle_mod, mode, M, N, K, seed=M + 5 * N + 3 * K)
    assert_gemm_close(oracle_mod, got, ref, absacc, f"{mode} {M}x{N}x{K}")


@pytest.mark.parametrize("mode,M,N,K,persistent", LARGE_M_SHAPES)
def test_gemm_large_m_full(oracle_mod, mode, M, N, K, persistent):
    plan = bw.gemm_plan(M, N, K, mode)
    assert plan["tiles"] > _sms() and plan["ksplit"] == 1
    assert (plan["ctas"] < plan["tiles"]) == persistent, plan
    got, ref, absacc = _gemm_case(oracle_mod, mode, M, N, K, seed=M + 3 * N + 7 * K)
    assert_gemm_close(oracle_mod, got, ref, absacc, f"{mode} {M}x{N}x{K}")


# ------------------------------------------------------------ invariants
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [16, 200])
def test_gemm_sign_symmetry_bitwise(mode, M):
    d = workloads.make(mode=mode, M=M, N=256, K=512, seed=M + 5)
    A = dev(d["A"].view(np.int16), torch.float16)
    s = dev(d["scales"].view(np.int16), torch.float16)
    pos = bw.lowbit_gemm(A, bw.pack(dev(d["codes"]), mode), s, mode)
    neg = bw.lowbit_gemm(A, bw.pack(dev(-d["codes"]), mode), s, mode)
    assert torch.equal(neg, -pos)


@pytest.mark.parametrize("mode", MODES)
def test_gemm_power_of_two_scaling_bitwise(mode):
    d = workloads.make(mode=mode, M=100, N=384, K=384, seed=77)
    A = dev(d["A"].view(np.int16), torch.float16)
    s = dev(d["scales"].view(np.int16), torch.float16)
    p = bw.pack(dev(d["codes"]), mode)
    one = bw.lowbit_gemm(A, p, s, mode)
    two = bw.lowbit_gemm(A * 2, p, s, mode)
    # Doubling commutes with every FP32 partial sum and with the final FP16
    # rounding, except where the result is FP16-subnormal (fixed 2^-24 grid).
    normal = one.abs() >= 2.0 ** -14
    assert normal.float().mean() > 0.99
    assert torch.equal(two[normal], one[normal] * 2)


@pytest.mark.parametrize("mode", MODES)
def test_gemm_all_ones_closed_form(oracle_mod, mode):
    N, K = 256, 1024
    rng = np.random.default_rng(99)
    c = workloads.codes(rng, N, K, mode)
    s = workloads.scales(rng, N, K)
    want = (c.reshape(N, K // 128, 128).astype(np.float64).sum(axis=2) *
            s.view(np.float16).astype(np.float64)).sum(axis=1)
    A = torch.ones((48, K), dtype=torch.float16, device="cuda")
    out = bw.lowbit_gemm(A, bw.pack(dev(c), mode), dev(s.view(np.int16), torch.float16), mode)
    got = out.double().cpu().numpy()
    absw = (np.abs(c).reshape(N, K // 128, 128).sum(axis=2) * s.view(np.float16).astype(np.float64)).sum(axis=1)
    ref_bits = oracle_mod.double_to_half_bits(want)
    tol = RTOL * absw + oracle_mod.ulp16(ref_bits)
    assert np.all(np.abs(got - want[None, :]) <= tol[None, :])


def test_gemm_rows_independent():
    d = workloads.make(mode="ternary", M=64, N=256, K=512, seed=3)
    A = dev(d["A"].view(np.int16), torch.float16)
    s = dev(d["scales"].view(np.int16), torch.float16)
    p = bw.pack(dev(d["codes"]), "ternary")
    base = bw.lowbit_gemm(A, p, s, "ternary")
    A2 = A.clone()
    A2[1:] = torch.randn_like(A2[1:])
    assert torch.equal(bw.lowbit_gemm(A2, p, s, "ternary")[0], base[0])


def test_gemm_matches_dequant_then_torch_matmul():
    """Secondary cross-check (not the oracle): GPU dequant -> fp32 matmul."""
    d = workloads.make(mode="ternary", M=300, N=512, K=1024, seed=8)
    A = dev(d["A"].view(np.int16), torch.float16)
    s = dev(d["scales"].view(np.int16), torch.float16)
    p = bw.pack(dev(d["codes"]), "ternary")
    W = bw.dequant(p, s, 1024, "ternary")
    ref = A.float() @ W.float().T
    got = bw.lowbit_gemm(A, p, s, "ternary").float()
    bound = 1e-3 * (A.float().abs() @ W.float().abs().T) + ref.abs() * 2.0 ** -10 + 2.0 ** -24
    assert bool(((got - ref).abs() <= bound).all())


# Narrow tiles with many groups per CTA: converters run up to one TMEM stage
# use ahead of the MMAs, so a wrong stage count would let a parity wait match
# an old phase (a timeout, or a stage overwritten while still read).  Many
# back-to-back launches give the race its chances.
@pytest.mark.parametrize("mode,M,N,K", [("ternary", 16, 3072, 12288), ("ternary", 32, 3072, 12288),
                                        ("ternary", 64, 3072, 12288), ("ternary", 64, 9216, 3072),
                                        ("binary", 64, 3072, 12288), ("ternary", 128, 3072, 12288),
                                        ("ternary_b3", 16, 3072, 12288), ("ternary_b3", 64, 9216, 3072)])
def test_narrow_tiles_repeated_launches(oracle_mod, mode, M, N, K):
    d = workloads.make(mode=mode, M=M, N=N, K=K, seed=M + N + K)
    ref_packed, packed, A, scales = gpu_inputs(d, oracle_mod)
    first = bw.lowbit_gemm(A, packed, scales, mode)
    out = torch.empty_like(first)
    torch.cuda.synchronize()
    for _ in range(150):
        bw.lowbit_gemm(A, packed, scales, mode, out=out)
    torch.cuda.synchronize()
    assert bw.get_device_error() == 0
    assert torch.equal(out, first)
    rng = np.random.default_rng(K)
    ms, ns = rng.integers(0, M, 600), rng.integers(0, N, 600)
    ref, _, absacc = oracle_mod.gemm_entries(d["A"], ref_packed, d["scales"], K, mode, ms, ns)
    assert_gemm_close(oracle_mod, to_u16(first)[ms, ns], ref, absacc, f"{mode} {M}x{N}x{K}")


# Host buffers in and out: chunked copies and GEMMs on the library's streams,
# ordered on the caller's stream.  Ragged M over several chunks, compared in
# full; the headline workload at sampled positions; back-to-back calls that
# reuse the same work buffers.
@pytest.mark.parametrize("mode,M,N,K", [("ternary", 1357, 3880, 512), ("binary", 16, 3072, 1024),
                                        ("ternary", 300, 256, 384), ("ternary_b3", 600, 384, 640)])
def test_gemm_host_buffers_full(oracle_mod, mode, M, N, K):
    d = workloads.make(mode=mode, M=M, N=N, K=K, seed=7 * M + N + K)
    ref_packed = oracle_mod.pack(d["codes"], mode)
    packed = bw.pack(dev(d["codes"]), mode)
    scales = dev(d["scales"].view(np.int16), torch.float16)
    A_host = torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).pin_memory()
    out_host = bw.lowbit_gemm_host(A_host, packed, scales, mode)
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.gemm(d["A"], ref_packed, d["scales"], K, mode)
    assert_gemm_close(oracle_mod, out_host.view(torch.int16).numpy().view(np.uint16), ref, absacc,
                      f"host buffers {mode} {M}x{N}x{K}")


def test_gemm_host_buffers_headline_and_reuse(oracle_mod):
    p = workloads.TERNARY_MLP_UP_4608
    d = workloads.make(p)
    ref_packed = oracle_mod.pack(d["codes"], p.mode)
    packed = bw.pack(dev(d["codes"]), p.mode)
    scales = dev(d["scales"].view(np.int16), torch.float16)
    A_host = torch.from_numpy(d["A"].view(np.int16)).view(torch.float16).pin_memory()
    A2_host = (A_host.float() * -2.0).half().pin_memory()  # exact: the output negates and doubles
    A_dev = torch.empty((p.M, p.K), dtype=torch.float16, device="cuda")
    out_dev = torch.empty((p.M, p.N), dtype=torch.float16, device="cuda")
    out1 = torch.empty((p.M, p.N), dtype=torch.float16).pin_memory()
    out2 = torch.empty((p.M, p.N), dtype=torch.float16).pin_memory()
    bw.lowbit_gemm_host(A_host, packed, scales, p.mode, out_host=out1, A_dev=A_dev, out_dev=out_dev)
    bw.lowbit_gemm_host(A2_host, packed, scales, p.mode, out_host=out2, A_dev=A_dev, out_dev=out_dev)
    torch.cuda.synchronize()
    assert bw.get_device_error() == 0
    got = out1.view(torch.int16).numpy().view(np.uint16)
    ms, ns = _sample_positions(p.M, p.N, 256, 3000, p.seed)
    ref, _, absacc = oracle_mod.gemm_entries(d["A"], ref_packed, d["scales"], p.K, p.mode, ms, ns)
    assert_gemm_close(oracle_mod, got[ms, ns], ref, absacc, "host buffers, headline workload")
    # The second call (same plans, same summation order) against the first,
    # exactly, through the scaling invariant: -2 scales the FP32 sum exactly
    # and commutes with rounding wherever the result is a normal FP16 number.
    normal = out1.float().abs() >= 2.0 ** -13
    assert bool(normal.float().mean() > 0.99)
    assert torch.equal(out2[normal], (out1.float() * -2.0).half()[normal])


# ------------------------------------------------- back-to-back launches
# Launches overlap their prologue with the previous kernel in the stream and
# wait for it before touching global memory; these check both hazards.
@pytest.mark.parametrize("M", [16, 4608])
def test_chained_layers_read_after_write(oracle_mod, M):
    K = 3072
    d1 = workloads.make(mode="ternary", M=M, N=K, K=K, seed=71)
    d2 = workloads.make(mode="binary", M=M, N=K, K=K, seed=72)
    A = dev(d1["A"].view(np.int16), torch.float16)
    p1, s1 = bw.pack(dev(d1["codes"]), "ternary"), dev(d1["scales"].view(np.int16), torch.float16)
    p2, s2 = bw.pack(dev(d2["codes"]), "binary"), dev(d2["scales"].view(np.int16), torch.float16)
    torch.cuda.synchronize()
    h1 = bw.lowbit_gemm(A, p1, s1, "ternary")
    h2 = bw.lowbit_gemm(h1, p2, s2, "binary")  # reads what the previous launch wrote
    torch.cuda.synchronize()
    h1_bits, h2_bits = to_u16(h1), to_u16(h2)
    rng = np.random.default_rng(M)
    ms, ns = rng.integers(0, M, 2000), rng.integers(0, K, 2000)
    ref, _, absacc = oracle_mod.gemm_entries(h1_bits, oracle_mod.pack(d2["codes"], "binary"), d2["scales"], K,
                                             "binary", ms, ns)
    assert_gemm_close(oracle_mod, h2_bits[ms, ns], ref, absacc, f"chained layer 2, M={M}")


def test_back_to_back_write_after_read(oracle_mod):
    M = N = K = 3072
    d = workloads.make(mode="ternary", M=M, N=N, K=K, seed=73)
    A = dev(d["A"].view(np.int16), torch.float16)
    packed, scales = bw.pack(dev(d["codes"]), "ternary"), dev(d["scales"].view(np.int16), torch.float16)
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    torch.cuda.synchronize()
    bw.lowbit_gemm(A, packed, scales, "ternary", out=out)
    bw.lowbit_gemm(out, packed, scales, "ternary", out=A)  # overwrites the input of the previous launch
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    ms, ns = rng.integers(0, M, 2000), rng.integers(0, N, 2000)
    ref, _, absacc = oracle_mod.gemm_entries(d["A"], oracle_mod.pack(d["codes"], "ternary"), d["scales"], K,
                                             "ternary", ms, ns)
    assert_gemm_close(oracle_mod, to_u16(out)[ms, ns], ref, absacc, "first launch after a dependent overwrite")


# ------------------------------------------------------------ edge cases
def test_gemm_empty_shapes():
    A = torch.zeros((0, 128), dtype=torch.float16, device="cuda")
    p = torch.zeros((8, 8), dtype=torch.int32, device="cuda")
    s = torch.zeros((8, 1), dtype=torch.float16, device="cuda")
    assert bw.lowbit_gemm(A, p, s, "ternary").shape == (0, 8)
    A = torch.ones((4, 0), dtype=torch.float16, device="cuda")
    out = bw.lowbit_gemm(A, torch.zeros((8, 0), dtype=torch.int32, device="cuda"),
                         torch.zeros((8, 0), dtype=torch.float16, device="cuda"), "ternary",
                         out=torch.full((4, 8), 7.0, dtype=torch.float16, device="cuda"))
    assert torch.equal(out, torch.zeros_like(out))


@pytest.mark.parametrize("mode", MODES)
def test_gemm_overflow_and_nan_match_the_oracle(oracle_mod, mode):
    """Outputs beyond the FP16 range round to +-inf on both sides; a NaN
    activation makes its whole output row NaN (every weight multiplies it)."""
    M, N, K = 24, 256, 512
    d = workloads.make(mode=mode, M=M, N=N, K=K, seed=31)
    A = d["A"].copy()
    A[:4] = np.float16(6.0e4).view(np.uint16)             # rows 0-3: huge activations -> overflow
    A[4:8] = np.float16(-6.0e4).view(np.uint16)
    A[8, 100] = np.uint16(0x7E00)                         # row 8: one NaN
    scales = d["scales"].copy()
    scales[:, :] = np.float16(0.5).view(np.uint16)
    ref_packed, packed, _, _ = gpu_inputs(d, oracle_mod)
    out = bw.lowbit_gemm(dev(A.view(np.int16), torch.float16), packed, dev(scales.view(np.int16), torch.float16),
                         mode)
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.gemm(A, ref_packed, scales, K, mode)
    got = to_u16(out)
    r = ref.view(np.float16)
    assert np.isinf(r[:8]).any() and np.isnan(r[8]).all()  # the case is what it claims
    assert_gemm_close(oracle_mod, got, ref, absacc, f"{mode} overflow / NaN")


def test_gemm_zero_codes_and_zero_scales():
    K = 384
    A = torch.randn((40, K), dtype=torch.float16, device="cuda")
    s = torch.rand((200, K // 128), dtype=torch.float16, device="cuda")
    z = bw.pack(torch.zeros((200, K), dtype=torch.int8, device="cuda"), "ternary")
    assert not bw.lowbit_gemm(A, z, s, "ternary").any()
    c = bw.pack(torch.ones((200, K), dtype=torch.int8, device="cuda"), "binary")
    assert not bw.lowbit_gemm(A, c, torch.zeros_like(s), "binary").any()


def test_misaligned_pointer_rejected():
    buf = torch.zeros(4 * 128 + 8, dtype=torch.float16, device="cuda")
    A = buf[1:1 + 4 * 128].view(4, 128)
    p = torch.zeros((8, 8), dtype=torch.int32, device="cuda")
    s = torch.zeros((8, 1), dtype=torch.float16, device="cuda")
    with pytest.raises(bw.BonsaiError) as e:
        bw.lowbit_gemm(A, p, s, "ternary")
    assert e.value.status == 3


def test_bounded_wait_gives_up_and_reports():
    assert bw.selftest_wait_timeout(2_000_000) == 7  # 2 ms, nobody arrives: BONSAI_ERR_TIMEOUT
    assert bw.get_device_error() == 0
    d = workloads.make(workloads.TERNARY_TINY)
    out = bw.lowbit_gemm(dev(d["A"].view(np.int16), torch.float16), bw.pack(dev(d["codes"]), "ternary"),
                         dev(d["scales"].view(np.int16), torch.float16), "ternary")
    torch.cuda.synchronize()
    assert out.isfinite().all()


# --------------------------------------- 4-bit group-affine weights (HQQ) --
# Reading of the pages' "4-bit HQQ" (unpinned by the pages): w =
# fp16(fp16(q - z) * s), groups of 64 along K.  Pack and dequant bit-exact,
# the GEMM within the same tolerance as the other formats.
def _hqq4_inputs(d):
    q = dev(d["q"])
    packed = bw.hqq4_pack(q)
    return (packed, dev(d["scales"].view(np.int16), torch.float16), dev(d["zeros"].view(np.int16), torch.float16),
            dev(d["A"].view(np.int16), torch.float16))


@pytest.mark.parametrize("N,K", PACK_SHAPES)
def test_hqq4_pack_and_dequant_bit_exact(oracle_mod, N, K):
    d = workloads.make_hqq4(1, N, K, seed=N + K)
    packed, s, z, _ = _hqq4_inputs(d)
    ref_packed = oracle_mod.hqq4_pack(d["q"])
    assert np.array_equal(to_u32(packed), ref_packed)
    got = bw.hqq4_dequant(packed, s, z, K)
    assert np.all(nan_aware_equal(to_u16(got), oracle_mod.hqq4_dequant(ref_packed, d["scales"], d["zeros"], K)))


def test_hqq4_dequant_special_values(oracle_mod):
    rng = np.random.default_rng(21)
    N, K = 4096, 128
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    s = rng.integers(0, 65536, (N, 2)).astype(np.uint16)  # every kind of FP16: subnormal, inf, NaN, -0
    z = rng.integers(0, 65536, (N, 2)).astype(np.uint16)
    ref_packed = oracle_mod.hqq4_pack(q)
    got = bw.hqq4_dequant(dev(ref_packed.view(np.int32)), dev(s.view(np.int16), torch.float16),
                          dev(z.view(np.int16), torch.float16), K)
    assert np.all(nan_aware_equal(to_u16(got), oracle_mod.hqq4_dequant(ref_packed, s, z, K)))


def test_hqq4_pack_reports_bad_values():
    q = np.full((64, 256), 3, np.uint8)
    q[17, 200] = 16
    with pytest.raises(bw.BonsaiError) as e:
        bw.hqq4_pack(dev(q))
    assert e.value.status == 4


@pytest.mark.parametrize("M,N,K", SMALL_SHAPES + [(1357, 3880, 512), (700, 1000, 640), (16, 3072, 12288),
                                   (1000, 3000, 1152), (2048, 3072, 2048)])
def test_hqq4_gemm_full(oracle_mod, M, N, K):
    d = workloads.make_hqq4(M, N, K, seed=M + 5 * N + K)
    packed, s, z, A = _hqq4_inputs(d)
    out = bw.hqq4_gemm(A, packed, s, z)
    torch.cuda.synchronize()
    ref, _, absacc = oracle_mod.hqq4_gemm(d["A"], oracle_mod.hqq4_pack(d["q"]), d["scales"], d["zeros"], K)
    assert_gemm_close(oracle_mod, to_u16(out), ref, absacc, f"hqq4 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(4608, 9216, 3072), (16, 3072, 9216)])
def test_hqq4_gemm_full_size_sampled(oracle_mod, M, N, K):
    d = workloads.make_hqq4(M, N, K, seed=77)
    packed, s, z, A = _hqq4_inputs(d)
    for _ in range(20):  # repeated launches: no device error, identical bits
        out = bw.hqq4_gemm(A, packed, s, z)
    first = bw.hqq4_gemm(A, packed, s, z)
    torch.cuda.synchronize()
    assert bw.get_device_error() == 0 and torch.equal(out, first)
    rng = np.random.default_rng(M)
    ms = np.unique(rng.integers(0, M, 48))
    ns = np.unique(rng.integers(0, N, 256))
    rows = oracle_mod.hqq4_dequant(oracle_mod.hqq4_pack(d["q"][ns]), d["scales"][ns], d["zeros"][ns], K)
    ref, _, absacc = oracle_mod.gemm_w16(d["A"][ms], rows)
    got = to_u16(first)[np.ix_(ms, ns)]
    assert_gemm_close(oracle_mod, got, ref, absacc, f"hqq4 {M}x{N}x{K} sampled")
    if M > 128:
        plan = bw.gemm_plan(M, N, K, "hqq4")
        assert plan["ctas"] < plan["tiles"], plan  # the persistent kernel
